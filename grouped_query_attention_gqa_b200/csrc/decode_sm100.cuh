// GQA decode step on sm_100a: one new query token per sequence against a packed,
// un-rotated KV cache (page "Qwen2 architecture introduction", aicoding.csdn.net,
// §4.1.3 closing paragraph: only the h_kv groups are cached, and the current
// position's K and V are appended each step; page "从 Qwen 1 到 Qwen 2", nxmr.cn,
// §2.4).  The query of sequence b sits at position p = seqlens[b] and attends to
// all seqlens[b] cached rows (positions 0 .. p-1).
//
// The step is bound by the HBM stream of the cache, so the design is about
// streaming, not arithmetic:
//  * plan_kernel   : prefix sums of seqlens -> packed row offsets (one CTA).
//  * split_kernel  : for each KV group u (and block of <= 8 query heads), the
//    flattened cache rows [0, N) are cut into P equal slices, one per warp, so
//    every warp streams the same number of bytes whatever the length mix.  A
//    warp walks its slice sequence by sequence and emits one partial
//    (running max m, sum l, unnormalised O) per (slice, sequence) piece.  The
//    piece of slice w and sequence b is stored in slot w + b: walking the two
//    partitions together, every piece raises w or b by one, so slots are unique
//    and there are at most P + B - 1 of them.
//    Each warp owns a 3-stage ring of 16-row blocks filled by 1-D bulk copies
//    (one row of K or V per lane, padded rows so ldmatrix is conflict-free).
//    K rows are rotated in registers (RoPE on load) with cos/sin advanced by
//    an angle-addition recurrence, re-anchored exactly every 64 blocks; the
//    g <= 8 query heads of the group share every K/V row read.  Scores and PV
//    use the warp-level bf16 tensor-core instruction with the key rows as the
//    M dimension, so the 7 or 8 heads fill the N = 8 dimension.
//  * combine_kernel: log-sum-exp merge of the pieces of each sequence.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "rope.cuh"
#include "sm100_ptx.cuh"

namespace gqa {
namespace decode {

using namespace ptx;

constexpr int ROWS = 16;        // cache rows per block (MMA M)
constexpr int NS = 3;           // ring stages per warp
constexpr int WARPS = 4;        // workers per CTA
constexpr int HB = 8;           // query heads per head block (MMA N)
constexpr int REANCHOR = 64;    // blocks between exact recomputations of the RoPE angles
constexpr int PLAN_THREADS = 1024;
constexpr int COMBINE_THREADS = 256;

template <int D>
struct Cfg {
    static constexpr int ROWB = D * 2 + 16;        // padded shared-memory row, bytes
    static constexpr int KV = ROWS * ROWB;         // one block of K (or V)
    static constexpr int STAGE = 2 * KV;
    static constexpr int WARP_BYTES = NS * STAGE;
    static constexpr int SMEM = WARPS * WARP_BYTES;
    static constexpr int KS = D / 16;              // 16-wide steps along d
    static constexpr int HALF_KS = D / 32;         // steps in the first half of d
    static constexpr int NF = 4 * HALF_KS;         // RoPE frequencies owned by one lane
    static constexpr int PART = 2 * HB + HB * D;   // floats per partial: m[8], l[8], O[8][D]
};

struct Params {
    const __nv_bfloat16* q;    // [B, h_q, D]
    const __nv_bfloat16* kc;   // [N, h_kv, D]
    const __nv_bfloat16* vc;   // [N, h_kv, D]
    __nv_bfloat16* out;        // [B, h_q, D]
    const int64_t* off;        // [B + 1] packed row offsets
    float* part;               // [(P + B) * h_kv * n_hb * PART]
    int B, h_q, h_kv, g, n_hb, P;
    float scale_log2;
    double theta;
    int* err;
};

// ---------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(PLAN_THREADS) plan_kernel(const int* __restrict__ seqlens,
                                                            int64_t* __restrict__ off, int B, int* err) {
    __shared__ int64_t warp_tot[PLAN_THREADS / 32];
    __shared__ int64_t carry;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) {
        carry = 0;
        off[0] = 0;
    }
    __syncthreads();
    for (int base = 0; base < B; base += PLAN_THREADS) {
        const int i = base + tid;
        int64_t s = 0;
        if (i < B) {
            const int v = seqlens[i];
            if (v <= 0) atomicOr(err, kErrBadSeqlen);
            s = v > 0 ? v : 0;
        }
        int64_t x = s;   // inclusive warp scan
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int64_t y = __shfl_up_sync(0xffffffffu, x, d);
            if (lane >= d) x += y;
        }
        if (lane == 31) warp_tot[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int64_t t = warp_tot[lane];
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int64_t y = __shfl_up_sync(0xffffffffu, t, d);
                if (lane >= d) t += y;
            }
            warp_tot[lane] = t;   // inclusive over warps
        }
        __syncthreads();
        const int64_t before = carry + (warp > 0 ? warp_tot[warp - 1] : 0);
        if (i < B) off[i + 1] = before + x;
        __syncthreads();
        if (tid == 0) carry += warp_tot[PLAN_THREADS / 32 - 1];
        __syncthreads();
    }
}

// Slice w of the flattened rows: [N*w/P, N*(w+1)/P).
__device__ __forceinline__ int64_t slice_start(int64_t N, int w, int P) { return (N * w) / P; }
// The slice that contains row r (0 <= r < N): the largest w with slice_start(w) <= r.
__device__ __forceinline__ int slice_of(int64_t r, int64_t N, int P) {
    return static_cast<int>(((r + 1) * P + N - 1) / N - 1);
}
// The sequence that contains packed row r (0 <= r < off[B]): the last b with off[b] <= r.
__device__ __forceinline__ int seq_of(const int64_t* off, int B, int64_t r) {
    int lo = 0, hi = B;   // invariant: off[lo] <= r < off[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (off[mid] <= r) lo = mid;
        else hi = mid;
    }
    return lo;
}

// Iterates the 16-row blocks of one slice, sequence by sequence.
struct BlockCursor {
    int b;
    int64_t r;        // first packed row of the current block
    int64_t seg_end;  // end of the current (slice, sequence) piece
    int64_t end;      // end of the slice
    bool done;
    __device__ void init(const int64_t* off, int B, int64_t start, int64_t e) {
        end = e;
        done = start >= e;
        if (done) return;
        b = seq_of(off, B, start);
        r = start;
        seg_end = min(end, off[b + 1]);
    }
    __device__ void next(const int64_t* off) {
        r += ROWS;
        if (r < seg_end) return;
        int64_t row = seg_end;
        while (row < end) {
            ++b;
            const int64_t se = min(end, off[b + 1]);
            if (se > row) {
                r = row;
                seg_end = se;
                return;
            }
        }
        done = true;
    }
};

// Rotate the bf16 pair-halves held in x (dims i, i+1 of the first half) and y (their partners).
__device__ __forceinline__ void rot_pair(uint32_t& x, uint32_t& y, float c0, float s0, float c1, float s1) {
    float a0, b0, a1, b1;
    rope_rotate(bf16lo_to_f32(x), bf16lo_to_f32(y), c0, s0, a0, b0);
    rope_rotate(bf16hi_to_f32(x), bf16hi_to_f32(y), c1, s1, a1, b1);
    x = pack_bf16x2(a0, a1);
    y = pack_bf16x2(b0, b1);
}

template <int D>
__global__ void __launch_bounds__(WARPS * 32) split_kernel(const Params p) {
    using C = Cfg<D>;
    constexpr int H = D / 2;
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint64_t bars[WARPS][NS];
    __shared__ double finv[H];
    __shared__ float2 rot8[H];   // cos/sin of 8 * f_i: the step between a lane's two rows of a block

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x / (p.h_kv * p.n_hb);
    const int gi = blockIdx.x % G;
    const int uh = blockIdx.x / G;
    const int u = uh / p.n_hb, hb = uh % p.n_hb;
    const int w = gi * WARPS + warp;

    for (int i = threadIdx.x; i < H; i += blockDim.x) {
        const double f = rope_inv_freq(i, D, p.theta);
        finv[i] = f;
        float c, s;
        rope_cossin(8.0, f, c, s);
        rot8[i] = make_float2(c, s);
    }
    if (lane == 0) {
        for (int s = 0; s < NS; ++s) mbar_init(&bars[warp][s], 1);
        fence_mbar_init();
    }
    __syncthreads();   // the last CTA-wide barrier: warps are independent from here on

    const int64_t N = p.off[p.B];
    const int64_t start = slice_start(N, w, p.P);
    const int64_t end = slice_start(N, w + 1, p.P);
    if (start >= end) return;

    uint8_t* wsm = smem + warp * C::WARP_BYTES;
    const uint32_t wsm_a = smem_u32(wsm);
    const int t4 = lane >> 2, tq = lane & 3;
    const size_t row_stride = static_cast<size_t>(p.h_kv) * D;

    // ---- producer side of the warp's ring
    BlockCursor iss;
    iss.init(p.off, p.B, start, end);
    auto issue = [&](int stage) {
        const int nvalid = static_cast<int>(iss.seg_end - iss.r < ROWS ? iss.seg_end - iss.r : ROWS);
        uint64_t* bar = &bars[warp][stage];
        if (lane == 0) mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nvalid * D * 2 * 2));
        __syncwarp();
        const int i = lane & (ROWS - 1);
        const bool is_v = lane >= ROWS;
        uint8_t* dst = wsm + stage * C::STAGE + (is_v ? C::KV : 0) + i * C::ROWB;
        fence_proxy_async_smem();
        if (i < nvalid) {
            const __nv_bfloat16* src = (is_v ? p.vc : p.kc) + (iss.r + i) * row_stride + static_cast<size_t>(u) * D;
            bulk_load(dst, src, D * 2, bar);
        } else {
#pragma unroll
            for (int c = 0; c < D / 8; ++c) reinterpret_cast<uint4*>(dst)[c] = make_uint4(0, 0, 0, 0);
        }
        iss.next(p.off);
    };
    for (int s = 0; s < NS && !iss.done; ++s) issue(s);

    // ---- consumer
    BlockCursor cur;
    cur.init(p.off, p.B, start, end);
    int kblk = 0;
    const float sl2 = p.scale_log2;
    while (!cur.done) {
        // ======== new piece: sequence cur.b, rows [cur.r, cur.seg_end)
        const int b = cur.b;
        const int64_t seq0 = p.off[b];
        const int64_t seg_end = cur.seg_end;
        const double qpos = static_cast<double>(p.off[b + 1] - seq0);   // query position = cache length

        // Q'^T as the B operand: lane holds head t4 of the block, dims 16ks + 2tq + {0,1} (b0) and +8 (b1).
        uint32_t qb[C::KS][2];
        {
            const int hl = hb * HB + t4;
            const bool valid = hl < p.g;
            const __nv_bfloat16* qrow = p.q + (static_cast<int64_t>(b) * p.h_q + u * p.g + (valid ? hl : 0)) * D;
#pragma unroll
            for (int ks = 0; ks < C::KS; ++ks) {
                const int d0 = 16 * ks + 2 * tq;
                qb[ks][0] = valid ? *reinterpret_cast<const uint32_t*>(qrow + d0) : 0u;
                qb[ks][1] = valid ? *reinterpret_cast<const uint32_t*>(qrow + d0 + 8) : 0u;
            }
#pragma unroll
            for (int ks = 0; ks < C::HALF_KS; ++ks) {
                const int d0 = 16 * ks + 2 * tq;
                float c[4], s[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) rope_cossin(qpos, finv[d0 + (e & 1) + 8 * (e >> 1)], c[e], s[e]);
                rot_pair(qb[ks][0], qb[ks + C::HALF_KS][0], c[0], s[0], c[1], s[1]);
                rot_pair(qb[ks][1], qb[ks + C::HALF_KS][1], c[2], s[2], c[3], s[3]);
            }
        }

        float o[C::KS][4];
#pragma unroll
        for (int mt = 0; mt < C::KS; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
        float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
        float ca[C::NF], sa[C::NF];   // cos/sin for the lane's first row of the block (row t4)
        int since_anchor = REANCHOR;

        while (!cur.done && cur.b == b) {
            const int stage = kblk % NS;
            mbar_wait(&bars[warp][stage], (kblk / NS) & 1, p.err, nullptr);
            __syncwarp();
            const int nvalid = static_cast<int>(seg_end - cur.r < ROWS ? seg_end - cur.r : ROWS);
            const int64_t jb = cur.r - seq0;   // position of the block's first row

            if (since_anchor >= REANCHOR) {
#pragma unroll
                for (int f = 0; f < C::NF; ++f) {
                    const int di = 16 * (f >> 2) + 2 * tq + (f & 1) + 8 * ((f >> 1) & 1);
                    rope_cossin(static_cast<double>(jb + t4), finv[di], ca[f], sa[f]);
                }
                since_anchor = 0;
            }
            // cos/sin for row t4 + 8
            float cb[C::NF], sb[C::NF];
#pragma unroll
            for (int f = 0; f < C::NF; ++f) {
                const int di = 16 * (f >> 2) + 2 * tq + (f & 1) + 8 * ((f >> 1) & 1);
                const float2 r8 = rot8[di];
                cb[f] = fmaf(ca[f], r8.x, -sa[f] * r8.y);
                sb[f] = fmaf(sa[f], r8.x, ca[f] * r8.y);
            }

            const uint32_t k_a = wsm_a + stage * C::STAGE;
            const uint32_t v_a = k_a + C::KV;
            // ---- S^T = K' Q'^T  (M = 16 rows, N = 8 heads, K = D)
            float sacc[4] = {0.f, 0.f, 0.f, 0.f};
            const uint32_t krow = k_a + ((lane & 7) + 8 * ((lane >> 3) & 1)) * C::ROWB + 8 * (lane >> 4) * 2;
#pragma unroll
            for (int ks = 0; ks < C::HALF_KS; ++ks) {
                uint32_t a[4], a2[4];
                ldsm_x4(krow + 16 * ks * 2, a[0], a[1], a[2], a[3]);
                ldsm_x4(krow + 16 * (ks + C::HALF_KS) * 2, a2[0], a2[1], a2[2], a2[3]);
                const int f = 4 * ks;
                rot_pair(a[0], a2[0], ca[f], sa[f], ca[f + 1], sa[f + 1]);           // row t4,   dims +0,+1
                rot_pair(a[1], a2[1], cb[f], sb[f], cb[f + 1], sb[f + 1]);           // row t4+8, dims +0,+1
                rot_pair(a[2], a2[2], ca[f + 2], sa[f + 2], ca[f + 3], sa[f + 3]);   // row t4,   dims +8,+9
                rot_pair(a[3], a2[3], cb[f + 2], sb[f + 2], cb[f + 3], sb[f + 3]);   // row t4+8, dims +8,+9
                mma_bf16_16816(sacc, a[0], a[1], a[2], a[3], qb[ks][0], qb[ks][1]);
                mma_bf16_16816(sacc, a2[0], a2[1], a2[2], a2[3], qb[ks + C::HALF_KS][0], qb[ks + C::HALF_KS][1]);
            }
            // advance the angles to the next block's first row (row t4 + 16)
#pragma unroll
            for (int f = 0; f < C::NF; ++f) {
                const int di = 16 * (f >> 2) + 2 * tq + (f & 1) + 8 * ((f >> 1) & 1);
                const float2 r8 = rot8[di];
                ca[f] = fmaf(cb[f], r8.x, -sb[f] * r8.y);
                sa[f] = fmaf(sb[f], r8.x, cb[f] * r8.y);
            }
            ++since_anchor;

            // ---- online softmax over the block (heads 2tq, 2tq+1 per lane; rows t4, t4+8)
            const bool v_lo = t4 < nvalid, v_hi = t4 + 8 < nvalid;
            const float x0 = v_lo ? sacc[0] * sl2 : -INFINITY;
            const float x1 = v_lo ? sacc[1] * sl2 : -INFINITY;
            const float x2 = v_hi ? sacc[2] * sl2 : -INFINITY;
            const float x3 = v_hi ? sacc[3] * sl2 : -INFINITY;
            float bm0 = fmaxf(x0, x2), bm1 = fmaxf(x1, x3);
#pragma unroll
            for (int sh = 4; sh < 32; sh <<= 1) {
                bm0 = fmaxf(bm0, __shfl_xor_sync(0xffffffffu, bm0, sh));
                bm1 = fmaxf(bm1, __shfl_xor_sync(0xffffffffu, bm1, sh));
            }
            const float mn0 = fmaxf(m0, bm0), mn1 = fmaxf(m1, bm1);
            const float al0 = ex2(m0 - mn0), al1 = ex2(m1 - mn1);
            m0 = mn0;
            m1 = mn1;
            const float p0 = ex2(x0 - m0), p1 = ex2(x1 - m1), p2 = ex2(x2 - m0), p3 = ex2(x3 - m1);
            l0 = fmaf(l0, al0, p0 + p2);
            l1 = fmaf(l1, al1, p1 + p3);
            const uint32_t pb0 = movmatrix_t(pack_bf16x2(p0, p1));   // P^T: keys 2tq,2tq+1 / head t4
            const uint32_t pb1 = movmatrix_t(pack_bf16x2(p2, p3));   // keys 8+2tq, 9+2tq

            // ---- O^T += V^T P^T  (M = 16 dims per tile, N = 8 heads, K = 16 rows)
            const uint32_t vrow = v_a + ((lane & 7) + 8 * (lane >> 4)) * C::ROWB + 8 * ((lane >> 3) & 1) * 2;
#pragma unroll
            for (int mt = 0; mt < C::KS; ++mt) {
                o[mt][0] *= al0;
                o[mt][1] *= al1;
                o[mt][2] *= al0;
                o[mt][3] *= al1;
                uint32_t v0, v1, v2, v3;
                ldsm_x4_t(vrow + 16 * mt * 2, v0, v1, v2, v3);
                mma_bf16_16816(o[mt], v0, v1, v2, v3, pb0, pb1);
            }
            __syncwarp();
            if (!iss.done) issue(stage);
            ++kblk;
            cur.next(p.off);
        }

        // ======== write the piece's partial into slot w + b
#pragma unroll
        for (int sh = 4; sh < 32; sh <<= 1) {
            l0 += __shfl_xor_sync(0xffffffffu, l0, sh);
            l1 += __shfl_xor_sync(0xffffffffu, l1, sh);
        }
        float* pp = p.part + ((static_cast<int64_t>(w + b) * p.h_kv + u) * p.n_hb + hb) * C::PART;
        if (lane < 4) {
            pp[2 * lane] = m0;
            pp[2 * lane + 1] = m1;
            pp[HB + 2 * lane] = l0;
            pp[HB + 2 * lane + 1] = l1;
        }
        float* po = pp + 2 * HB;
#pragma unroll
        for (int mt = 0; mt < C::KS; ++mt) {
            const int d = 16 * mt + t4;
            po[(2 * tq) * D + d] = o[mt][0];
            po[(2 * tq + 1) * D + d] = o[mt][1];
            po[(2 * tq) * D + d + 8] = o[mt][2];
            po[(2 * tq + 1) * D + d + 8] = o[mt][3];
        }
    }
}

// ---------------------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(COMBINE_THREADS) combine_kernel(const Params p) {
    using C = Cfg<D>;
    __shared__ float sM[HB], sInvL[HB];
    const int hb = blockIdx.x % p.n_hb;
    const int u = (blockIdx.x / p.n_hb) % p.h_kv;
    const int b = blockIdx.x / (p.n_hb * p.h_kv);
    const int nh = min(HB, p.g - hb * HB);
    const int64_t N = p.off[p.B];
    const int64_t s0 = p.off[b], s1 = p.off[b + 1];
    __nv_bfloat16* ob = p.out + (static_cast<int64_t>(b) * p.h_q + u * p.g + hb * HB) * D;
    if (s1 <= s0) {   // empty (invalid) sequence: zeros, flagged by plan_kernel
        for (int e = threadIdx.x; e < nh * D; e += blockDim.x) ob[e] = __float2bfloat16(0.f);
        return;
    }
    const int w_lo = slice_of(s0, N, p.P);
    const int w_hi = slice_of(s1 - 1, N, p.P);
    auto part_of = [&](int w) {
        return p.part + ((static_cast<int64_t>(w + b) * p.h_kv + u) * p.n_hb + hb) * C::PART;
    };
    // Slices strictly inside (w_lo, w_hi) may be empty when N < P: they wrote nothing.
    auto empty = [&](int w) { return slice_start(N, w + 1, p.P) <= slice_start(N, w, p.P); };
    if (threadIdx.x < nh) {
        const int h = threadIdx.x;
        float M = -INFINITY;
        for (int w = w_lo; w <= w_hi; ++w)
            if (!empty(w)) M = fmaxf(M, part_of(w)[h]);
        float L = 0.f;
        for (int w = w_lo; w <= w_hi; ++w) {
            if (empty(w)) continue;
            const float* pp = part_of(w);
            L += pp[HB + h] * ex2(pp[h] - M);
        }
        sM[h] = M;
        sInvL[h] = 1.0f / L;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < nh * D; e += blockDim.x) {
        const int h = e / D, d = e % D;
        float acc = 0.f;
        for (int w = w_lo; w <= w_hi; ++w) {
            if (empty(w)) continue;
            const float* pp = part_of(w);
            acc += pp[2 * HB + h * D + d] * ex2(pp[h] - sM[h]);
        }
        ob[e] = __float2bfloat16(acc * sInvL[h]);
    }
}

}  // namespace decode
}  // namespace gqa

// GQA decode step on sm_100a: one new query token per sequence against a packed,
// un-rotated KV cache (page "Qwen2 architecture introduction", aicoding.csdn.net,
// §4.1.3 closing paragraph: only the h_kv groups are cached, and the current
// position's K and V are appended each step; page "从 Qwen 1 到 Qwen 2", nxmr.cn,
// §2.4).  The query of sequence b sits at position p = seqlens[b] and attends to
// all seqlens[b] cached rows (positions 0 .. p-1).
//
// The step streams the whole cache from HBM once, so the design is about streaming:
//  * plan_kernel   : prefix sums of seqlens -> packed row offsets (one CTA).
//  * split_kernel  : for each KV group u (and block of <= 8 query heads), the
//    flattened cache rows [0, N) are cut into P equal slices, one per warp, so
//    every warp streams the same number of bytes whatever the length mix.  A
//    warp walks its slice sequence by sequence and emits one partial
//    (running max m, sum l, unnormalised O) per (slice, sequence) piece.  The
//    piece of slice w and sequence b is stored in slot w + b: walking the two
//    partitions together, every piece raises w or b by one, so slots are unique
//    and there are at most P + B - 1 of them.
//    Each warp owns a 2-stage ring of 16-row blocks filled by 1-D bulk copies
//    (one row of K or V per lane, padded rows so ldmatrix is conflict-free).
//    K rows are rotated in registers (RoPE on load) with cos/sin advanced by
//    an angle-addition recurrence, re-anchored exactly every 64 blocks; that
//    rotation is most of a block's instructions, enough to make the kernel
//    follow the SM clock once it drops under the power cap.  Over a cache that
//    keeps its keys after RoPE (KROT) the rows are used as loaded and the
//    kernel stays at the HBM stream.  The g <= 8 query heads of the group share
//    every K/V row read.  Scores and PV
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

#ifndef GQA_DECODE_STAGES
#define GQA_DECODE_STAGES 2
#endif
#ifndef GQA_PAGED_TRACK
#define GQA_PAGED_TRACK 1
#endif
#ifndef GQA_DECODE_CTAS_PER_SM
#define GQA_DECODE_CTAS_PER_SM 3
#endif
constexpr int ROWS = 16;        // cache rows per block (MMA M)
constexpr int NS = GQA_DECODE_STAGES;             // ring stages per warp
constexpr int WARPS = 4;        // workers per CTA
constexpr int CTAS_PER_SM = GQA_DECODE_CTAS_PER_SM;
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
    static constexpr int NP = NF / 2;              // ... as pairs of adjacent frequencies
    static constexpr int PART = 2 * HB + HB * D;   // floats per partial: m[8], l[8], O[8][D]
};

struct Params {
    const __nv_bfloat16* q;    // [B, h_q, D]
    const __nv_bfloat16* kc;   // packed: [N, h_kv, D]; paged: [num_pages * page_size, h_kv, D]
    const __nv_bfloat16* vc;   // same layout as kc
    const int* bt;             // paged only: block table [B, max_pages]; nullptr for the packed layout
    int page_size, max_pages, num_pages;
    __nv_bfloat16* out;        // [B, h_q, D]
    const int64_t* off;        // [B + 1] packed row offsets
    float* part;               // [(P + B) * h_kv * n_hb * PART]
    int B, h_q, h_kv, g, n_hb, P;
    int self_in_cache;         // 1: the cache already holds the query's own row; it sits at seqlens[b] - 1
    float scale_log2;
    RopeSpec rope;             // RoPE base and YaRN scaling (its temperature is in scale_log2)
    int* err;
};

// ---------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(PLAN_THREADS) plan_kernel(const int* __restrict__ seqlens,
                                                            int64_t* __restrict__ off, int B, int* err) {
    __shared__ int64_t warp_tot[PLAN_THREADS / 32];
    __shared__ int64_t carry;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // The split kernel may launch now: it waits for this grid's offsets with griddepcontrol.wait.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
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

// Rotate two adjacent first-half dims (bf16x2 word x) against their partners d + D/2 (word y), with
// (cos, sin) of the two frequencies as fp32 pairs C and S.
__device__ __forceinline__ void rot_pair(uint32_t& x, uint32_t& y, uint64_t C, uint64_t S) {
    const uint64_t X = f2_from_bf16x2(x), Y = f2_from_bf16x2(y);
    x = f2_to_bf16x2(f2_sub(f2_mul(X, C), f2_mul(Y, S)));
    y = f2_to_bf16x2(f2_fma(Y, C, f2_mul(X, S)));
}

// (C, S) <- (C, S) rotated by the angle with cosine / sine pairs (Cr, Sr): the angle-addition step.
__device__ __forceinline__ void rot_step(uint64_t& C, uint64_t& S, uint64_t Cr, uint64_t Sr) {
    const uint64_t c2 = f2_sub(f2_mul(C, Cr), f2_mul(S, Sr));
    S = f2_fma(S, Cr, f2_mul(C, Sr));
    C = c2;
}

// PAGED: cache rows are read through the block table p.bt (gqa_decode_paged); otherwise packed.
// KROT: the cached keys are already rotated at their positions (a cache that keeps keys after RoPE), so
// they go to the dot product as loaded; otherwise each key is rotated on load at its row index.
template <int D, bool PAGED, bool KROT>
__global__ void __launch_bounds__(WARPS * 32, CTAS_PER_SM) split_kernel(const Params p) {
    using C = Cfg<D>;
    constexpr int H = D / 2;
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint64_t bars[WARPS][NS];
    __shared__ double finv[H];
    // cos/sin of 8 * f_i for i, i+1 (i even) as {cos_i, cos_i+1, sin_i, sin_i+1}: the angle step between
    // a lane's two rows of a block, loaded as two fp32 pairs by one 128-bit read.
    __shared__ float4 rot8[H / 2];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x / (p.h_kv * p.n_hb);
    const int gi = blockIdx.x % G;
    const int uh = blockIdx.x / G;
    const int u = uh / p.n_hb, hb = uh % p.n_hb;
    const int w = gi * WARPS + warp;

    for (int i = threadIdx.x; i < H; i += blockDim.x) finv[i] = rope_freq(i, D, p.rope);
    for (int i = threadIdx.x; i < H / 2; i += blockDim.x) {
        float c0, s0, c1, s1;
        rope_cossin(8.0, rope_freq(2 * i, D, p.rope), c0, s0);
        rope_cossin(8.0, rope_freq(2 * i + 1, D, p.rope), c1, s1);
        rot8[i] = make_float4(c0, c1, s0, s1);
    }
    if (lane == 0) {
        for (int s = 0; s < NS; ++s) mbar_init(&bars[warp][s], 1);
        fence_mbar_init();
    }
    __syncthreads();   // the last CTA-wide barrier: warps are independent from here on
    // Launched as a programmatic dependent of plan_kernel: everything above overlaps it; the offsets it
    // writes are read only after its grid has completed.  The combine kernel may launch from here on.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    const int64_t N = p.off[p.B];
    const int64_t start = slice_start(N, w, p.P);
    const int64_t end = slice_start(N, w + 1, p.P);
    if (start >= end) return;

    uint8_t* wsm = smem + warp * C::WARP_BYTES;
    const uint32_t wsm_a = smem_u32(wsm);
    const int t4 = lane >> 2, tq = lane & 3;
    const size_t row_stride = static_cast<size_t>(p.h_kv) * D;

    // ---- producer side of the warp's ring.  Every cache row is read once: evict-first in L2.
    const uint64_t stream_policy = l2_evict_first_policy();
    BlockCursor iss;
    iss.init(p.off, p.B, start, end);
#if GQA_PAGED_TRACK
    // Paged, pages of >= 16 rows: the producer's current piece (sequence pg_b), the page index and offset
    // of its block's first row, and the table entries of that page and the next (-1: past the table).
    int pg_b = -1, pg_idx = 0, pg_rem = 0, pg_cur = -1, pg_next = -1;
    auto table_entry = [&](int b, int pi) {
        return pi < p.max_pages ? __ldg(p.bt + static_cast<int64_t>(b) * p.max_pages + pi) : -1;
    };
#endif
    auto issue = [&](int stage) {
        const int nvalid = static_cast<int>(iss.seg_end - iss.r < ROWS ? iss.seg_end - iss.r : ROWS);
        uint64_t* bar = &bars[warp][stage];
        const int i = lane & (ROWS - 1);
        const bool is_v = lane >= ROWS;
        // Storage row of logical row iss.r + i: the packed row itself, or its page slot through the block
        // table.  A table entry outside [0, num_pages), or a row past max_pages pages, is not read: the
        // row stays zero and the device error word gets kErrBadPage.
        bool load = i < nvalid;
        int64_t srow = iss.r + i;
#if GQA_PAGED_TRACK
        if (PAGED && p.page_size >= ROWS) {
            // Pages of at least 16 rows: a block spans at most two of them.  The block's page and the next
            // one are tracked from block to block (the next table entry read one page ahead), so a block
            // costs no division and no table read on its path.
            const int ps = p.page_size;
            if (iss.b != pg_b) {   // a new piece: locate its first block once (warp-uniform)
                pg_b = iss.b;
                const int j0 = static_cast<int>(iss.r - p.off[iss.b]);   // position in the sequence (< 2^31)
                pg_idx = j0 / ps;
                pg_rem = j0 - pg_idx * ps;
                pg_cur = table_entry(pg_b, pg_idx);
                pg_next = table_entry(pg_b, pg_idx + 1);
            } else {
                pg_rem += ROWS;
                if (pg_rem >= ps) {
                    pg_rem -= ps;
                    ++pg_idx;
                    pg_cur = pg_next;
                    pg_next = table_entry(pg_b, pg_idx + 1);
                }
            }
            const int t = pg_rem + i;
            const int page = t < ps ? pg_cur : pg_next;
            if (load) {
                if (page < 0 || page >= p.num_pages) {
                    load = false;
                    atomicOr(p.err, kErrBadPage);
                } else {
                    srow = static_cast<int64_t>(page) * ps + (t < ps ? t : t - ps);
                }
            }
        } else
#endif
        if (PAGED && load) {
            const int j = static_cast<int>(srow - p.off[iss.b]);   // position in the sequence (< 2^31)
            const int pi = j / p.page_size;
            const int page = pi < p.max_pages ? p.bt[static_cast<int64_t>(iss.b) * p.max_pages + pi] : -1;
            if (page < 0 || page >= p.num_pages) {
                load = false;
                atomicOr(p.err, kErrBadPage);
            } else {
                srow = static_cast<int64_t>(page) * p.page_size + (j - pi * p.page_size);
            }
        }
        // Arm the stage with the bytes of the rows that are really copied.
        const uint32_t nload = __popc(__ballot_sync(0xffffffffu, load));
        if (lane == 0) mbar_arrive_expect_tx(bar, nload * static_cast<uint32_t>(D * 2));
        __syncwarp();
        uint8_t* dst = wsm + stage * C::STAGE + (is_v ? C::KV : 0) + i * C::ROWB;
        fence_proxy_async_smem();
        if (load) {
            const __nv_bfloat16* src = (is_v ? p.vc : p.kc) + srow * row_stride + static_cast<size_t>(u) * D;
            bulk_load_hint(dst, src, D * 2, bar, stream_policy);
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
        // query position: the cache length, or its last row when that row is the query's own
        const double qpos = static_cast<double>(p.off[b + 1] - seq0 - p.self_in_cache);

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
                rot_pair(qb[ks][0], qb[ks + C::HALF_KS][0], f2_pack(c[0], c[1]), f2_pack(s[0], s[1]));
                rot_pair(qb[ks][1], qb[ks + C::HALF_KS][1], f2_pack(c[2], c[3]), f2_pack(s[2], s[3]));
            }
        }

        float o[C::KS][4];
#pragma unroll
        for (int mt = 0; mt < C::KS; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
        float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
        // cos/sin for the lane's first row of the block (row t4), as fp32 pairs of adjacent frequencies:
        // pair 2ks holds dims 16ks + 2tq + {0, 1}, pair 2ks + 1 holds dims 16ks + 2tq + 8 + {0, 1}.
        uint64_t ca[C::NP], sa[C::NP];
        int since_anchor = REANCHOR;

        while (!cur.done && cur.b == b) {
            const int stage = kblk % NS;
            mbar_wait(&bars[warp][stage], (kblk / NS) & 1, p.err, nullptr);
            __syncwarp();
            const int nvalid = static_cast<int>(seg_end - cur.r < ROWS ? seg_end - cur.r : ROWS);
            const int64_t jb = cur.r - seq0;   // position of the block's first row

            if (!KROT && since_anchor >= REANCHOR) {
#pragma unroll
                for (int fp = 0; fp < C::NP; ++fp) {
                    const int di = 16 * (fp >> 1) + 2 * tq + 8 * (fp & 1);
                    float c0, s0, c1, s1;
                    rope_cossin(static_cast<double>(jb + t4), finv[di], c0, s0);
                    rope_cossin(static_cast<double>(jb + t4), finv[di + 1], c1, s1);
                    ca[fp] = f2_pack(c0, c1);
                    sa[fp] = f2_pack(s0, s1);
                }
                since_anchor = 0;
            }
            const uint32_t k_a = wsm_a + stage * C::STAGE;
            const uint32_t v_a = k_a + C::KV;
            // ---- S^T = K' Q'^T  (M = 16 rows, N = 8 heads, K = D), two independent accumulator chains.
            // Per 16-wide step: cos/sin of row t4 + 8 from those of row t4 (one angle-addition step),
            // rotate both rows, then advance row t4's angles to row t4 + 16 for the next block.
            float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            const uint32_t krow = k_a + ((lane & 7) + 8 * ((lane >> 3) & 1)) * C::ROWB + 8 * (lane >> 4) * 2;
#pragma unroll
            for (int ks = 0; ks < C::HALF_KS; ++ks) {
                uint32_t a[4], a2[4];
                ldsm_x4(krow + 16 * ks * 2, a[0], a[1], a[2], a[3]);
                ldsm_x4(krow + 16 * (ks + C::HALF_KS) * 2, a2[0], a2[1], a2[2], a2[3]);
#pragma unroll
                for (int hf = 0; hf < (KROT ? 0 : 2); ++hf) {   // dims 16ks + 2tq + 8*hf + {0, 1}
                    const int fp = 2 * ks + hf;
                    const float4 r8 = rot8[(16 * ks + 2 * tq + 8 * hf) >> 1];
                    const uint64_t Cr = f2_pack(r8.x, r8.y), Sr = f2_pack(r8.z, r8.w);
                    uint64_t cb = ca[fp], sb = sa[fp];
                    rot_step(cb, sb, Cr, Sr);                       // row t4 + 8
                    rot_pair(a[2 * hf], a2[2 * hf], ca[fp], sa[fp]);          // row t4
                    rot_pair(a[2 * hf + 1], a2[2 * hf + 1], cb, sb);          // row t4 + 8
                    ca[fp] = cb;
                    sa[fp] = sb;
                    rot_step(ca[fp], sa[fp], Cr, Sr);               // row t4 + 16: next block's first row
                }
                mma_bf16_16816(sacc[0], a[0], a[1], a[2], a[3], qb[ks][0], qb[ks][1]);
                mma_bf16_16816(sacc[1], a2[0], a2[1], a2[2], a2[3], qb[ks + C::HALF_KS][0], qb[ks + C::HALF_KS][1]);
            }
            ++since_anchor;

            // ---- online softmax over the block (heads 2tq, 2tq+1 per lane; rows t4, t4+8)
            const bool v_lo = t4 < nvalid, v_hi = t4 + 8 < nvalid;
            const float x0 = v_lo ? (sacc[0][0] + sacc[1][0]) * sl2 : -INFINITY;
            const float x1 = v_lo ? (sacc[0][1] + sacc[1][1]) * sl2 : -INFINITY;
            const float x2 = v_hi ? (sacc[0][2] + sacc[1][2]) * sl2 : -INFINITY;
            const float x3 = v_hi ? (sacc[0][3] + sacc[1][3]) * sl2 : -INFINITY;
            float bm0 = fmaxf(x0, x2), bm1 = fmaxf(x1, x3);
#pragma unroll
            for (int sh = 4; sh < 32; sh <<= 1) {
                bm0 = fmaxf(bm0, __shfl_xor_sync(0xffffffffu, bm0, sh));
                bm1 = fmaxf(bm1, __shfl_xor_sync(0xffffffffu, bm1, sh));
            }
            const float mn0 = fmaxf(m0, bm0), mn1 = fmaxf(m1, bm1);
            const float al0 = ex2(m0 - mn0), al1 = ex2(m1 - mn1);
            // Once a sequence's running maximum settles it rarely grows: the rescale of O below is then a
            // multiplication by exactly 1 in every lane, and is skipped (the result is the same bit for bit).
            const bool grew = __any_sync(0xffffffffu, (mn0 > m0) | (mn1 > m1));
            m0 = mn0;
            m1 = mn1;
            const float p0 = ex2(x0 - m0), p1 = ex2(x1 - m1), p2 = ex2(x2 - m0), p3 = ex2(x3 - m1);
            l0 = fmaf(l0, al0, p0 + p2);
            l1 = fmaf(l1, al1, p1 + p3);
            const uint32_t pb0 = movmatrix_t(pack_bf16x2(p0, p1));   // P^T: keys 2tq,2tq+1 / head t4
            const uint32_t pb1 = movmatrix_t(pack_bf16x2(p2, p3));   // keys 8+2tq, 9+2tq

            // ---- O^T += V^T P^T  (M = 16 dims per tile, N = 8 heads, K = 16 rows)
            const uint32_t vrow = v_a + ((lane & 7) + 8 * (lane >> 4)) * C::ROWB + 8 * ((lane >> 3) & 1) * 2;
            if (grew) {
#pragma unroll
                for (int mt = 0; mt < C::KS; ++mt) {
                    o[mt][0] *= al0;
                    o[mt][1] *= al1;
                    o[mt][2] *= al0;
                    o[mt][3] *= al1;
                }
            }
#pragma unroll
            for (int mt = 0; mt < C::KS; ++mt) {
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
// One CTA per (sequence, KV group, head block).  The pieces of the sequence are processed CHUNK at a
// time: one thread per piece reads its (m, l) for the 8 heads, warp h reduces head h over the chunk
// (max, then the rescaled sum), and each thread accumulates 4 of the 8 x D outputs over the pieces with
// several loads in flight.
template <int D>
__global__ void __launch_bounds__(COMBINE_THREADS) combine_kernel(const Params p) {
    using C = Cfg<D>;
    constexpr int CHUNK = COMBINE_THREADS;   // pieces per round
    constexpr int PER_T = HB * D / COMBINE_THREADS;
    static_assert(COMBINE_THREADS == 32 * HB, "one warp per head");
    static_assert(HB * D % COMBINE_THREADS == 0, "outputs split evenly");
    __shared__ float s_m[CHUNK][HB + 1];
    __shared__ float s_l[CHUNK][HB + 1];
    __shared__ const float* s_ptr[CHUNK];
    __shared__ float s_M[HB], s_L[HB];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // A programmatic dependent of split_kernel: its partials are read only after its grid has completed.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int hb = blockIdx.x % p.n_hb;
    const int u = (blockIdx.x / p.n_hb) % p.h_kv;
    const int b = blockIdx.x / (p.n_hb * p.h_kv);
    const int nh = min(HB, p.g - hb * HB);
    const int64_t N = p.off[p.B];
    const int64_t s0 = p.off[b], s1 = p.off[b + 1];
    __nv_bfloat16* ob = p.out + (static_cast<int64_t>(b) * p.h_q + u * p.g + hb * HB) * D;
    if (s1 <= s0) {   // empty (invalid) sequence: zeros, flagged by plan_kernel
        for (int e = tid; e < nh * D; e += blockDim.x) ob[e] = __float2bfloat16(0.f);
        return;
    }
    const int w_lo = slice_of(s0, N, p.P);
    const int w_hi = slice_of(s1 - 1, N, p.P);
    // Pass 1: merged max M and sum L per head.  Slices strictly inside (w_lo, w_hi) may be empty when
    // N < P: they wrote nothing and are skipped.
    float M = -INFINITY, L = 0.f;   // warp `warp` tracks head `warp`
    for (int w0 = w_lo; w0 <= w_hi; w0 += CHUNK) {
        const int w = w0 + tid;
        const bool live = w <= w_hi && slice_start(N, w + 1, p.P) > slice_start(N, w, p.P);
        const float* pp = live ? p.part + ((static_cast<int64_t>(w + b) * p.h_kv + u) * p.n_hb + hb) * C::PART
                               : nullptr;
        s_ptr[tid] = pp;
#pragma unroll
        for (int h = 0; h < HB; ++h) {
            s_m[tid][h] = live ? pp[h] : -INFINITY;
            s_l[tid][h] = live ? pp[HB + h] : 0.f;
        }
        __syncthreads();
        float m = -INFINITY;
        for (int i = lane; i < CHUNK; i += 32) m = fmaxf(m, s_m[i][warp]);
#pragma unroll
        for (int sh = 16; sh > 0; sh >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, sh));
        const float Mn = fmaxf(M, m);
        float l = 0.f;
        for (int i = lane; i < CHUNK; i += 32) l += s_l[i][warp] * ex2(s_m[i][warp] - Mn);
#pragma unroll
        for (int sh = 16; sh > 0; sh >>= 1) l += __shfl_xor_sync(0xffffffffu, l, sh);
        L = L * ex2(M - Mn) + l;
        M = Mn;
        __syncthreads();
    }
    if (lane == 0) {
        s_M[warp] = M;
        s_L[warp] = L;
    }
    __syncthreads();
    // Pass 2: O = sum over pieces of O_piece * 2^(m_piece - M) / L.
    float acc[PER_T];
#pragma unroll
    for (int k = 0; k < PER_T; ++k) acc[k] = 0.f;
    for (int w0 = w_lo; w0 <= w_hi; w0 += CHUNK) {
        const int w = w0 + tid;
        const bool live = w <= w_hi && slice_start(N, w + 1, p.P) > slice_start(N, w, p.P);
        const float* pp = live ? p.part + ((static_cast<int64_t>(w + b) * p.h_kv + u) * p.n_hb + hb) * C::PART
                               : nullptr;
        s_ptr[tid] = pp;
#pragma unroll
        for (int h = 0; h < HB; ++h) s_m[tid][h] = live ? ex2(pp[h] - s_M[h]) / s_L[h] : 0.f;   // weights
        __syncthreads();
        const int n = min(CHUNK, w_hi - w0 + 1);
#pragma unroll 4
        for (int i = 0; i < n; ++i) {
            const float* po = s_ptr[i];
            if (po == nullptr) continue;
            po += 2 * HB;
#pragma unroll
            for (int k = 0; k < PER_T; ++k) {
                const int e = tid + k * COMBINE_THREADS;
                acc[k] = fmaf(po[e], s_m[i][e / D], acc[k]);
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int k = 0; k < PER_T; ++k) {
        const int e = tid + k * COMBINE_THREADS;
        if (e < nh * D) ob[e] = __float2bfloat16(acc[k]);
    }
}

}  // namespace decode
}  // namespace gqa

// libgqa: the C ABI declared in include/gqa.h.  Host-side validation, workspace
// management, tensor-map encoding and kernel launches.  All kernels live in the
// headers included below, so this is the library's single translation unit.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <numeric>
#include <set>
#include <utility>
#include <vector>

#include "../../include/gqa.h"
#include "decode_sm100.cuh"
#include "prefill_sm100.cuh"
#include "qkv_sm100.cuh"

namespace {

constexpr int kMaxDevices = 64;

// The device error word (GQA_DEVERR_* bits), one per device context.
__device__ int g_dev_err;

struct DeviceState {
    bool checked = false;
    bool supported = false;
    int num_sms = 0;
    int* err = nullptr;           // device address of g_dev_err
    void* ws = nullptr;           // prefill workspace
    size_t ws_bytes = 0;
    void* dws = nullptr;          // decode workspace
    size_t dws_bytes = 0;
    void* fixed_scratch = nullptr;   // device address of g_fixed_scratch (gqa_decode_noalloc)
    bool attn_ready[2] = {false, false};   // attention kernel attributes set and checked (d = 64, 128)
    // The tensor maps of the last prefill call, reused while every pointer and size matches.
    struct MapKey {
        const void *qr, *kr, *v, *out;
        int B, L, h_q, h_kv, d;
        bool operator==(const MapKey& o) const {
            return qr == o.qr && kr == o.kr && v == o.v && out == o.out && B == o.B && L == o.L && h_q == o.h_q &&
                   h_kv == o.h_kv && d == o.d;
        }
    } map_key{};
    bool maps_valid = false;
    CUtensorMap maps[4];
    // The attention kernel's work schedule for the last (B, L, h_q, h_kv, grid): per-CTA item lists (CSR).
    int sched_key[5] = {0, 0, 0, 0, 0};
    bool sched_valid = false;
    void* sched = nullptr;
    size_t sched_bytes = 0;
    // QKV projection: the cos / sin table of the last (L, d, theta), and the last pair of tensor maps.
    void* tab = nullptr;
    size_t tab_bytes = 0;
    int tab_L = -1, tab_d = 0;
    float tab_theta = 0.f, tab_factor = 1.f;
    int tab_orig = 0;
    unsigned gemm_ready = 0;   // bit per GEMM kernel instantiation whose shared-memory size is set
    const void* qkv_key[2] = {nullptr, nullptr};
    long long qkv_dims[4] = {0, 0, 0, 0};
    CUtensorMap qkv_maps[3];
    const void* proj_key[2] = {nullptr, nullptr};
    long long proj_dims[4] = {0, 0, 0, 0};
    CUtensorMap proj_maps[3];
    const void* app_key[2] = {nullptr, nullptr};
    long long app_dims[4] = {0, 0, 0, 0};
    CUtensorMap app_maps[3];
};

DeviceState g_dev[kMaxDevices];
cudaStream_t g_stream = nullptr;
cudaEvent_t g_ev_start = nullptr, g_ev_stop = nullptr;   // optional timing of the main kernel

// Decode query position for every later decode call (gqa_set_decode_self_in_cache): 0 = at seqlens[b],
// 1 = at seqlens[b] - 1, the cache's last row being the query's own.
int g_self_in_cache = 0;

// Whether the decode caches keep their keys after RoPE (gqa_set_decode_cache_rotated): 0 = raw keys, rotated
// on load by the decode; 1 = keys already rotated at their positions (with the YaRN temperature), written so
// by gqa_qkv_rope's k output and by gqa_qkv_append.
int g_cache_rotated = 0;

// YaRN scaling of RoPE for every later call (gqa_set_rope_scaling); factor 1 = plain RoPE.
float g_rope_factor = 1.0f;
int g_rope_orig = 0;

gqa::RopeSpec rope_spec(float theta) {
    return gqa::RopeSpec{std::log2(static_cast<double>(theta)), g_rope_factor > 1.0f ? static_cast<double>(g_rope_factor) : 1.0,
                    static_cast<double>(g_rope_orig)};
}
// YaRN's temperature on each rotated row: the logits scale by its square.
float rope_mscale() { return g_rope_factor > 1.0f ? static_cast<float>(0.1 * std::log(g_rope_factor) + 1.0) : 1.0f; }

inline void mark(cudaEvent_t ev) {
    if (g_ev_start && g_ev_stop) cudaEventRecord(ev, g_stream);
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

// Current device's state, after a one-time check that it is an sm_100 part.
DeviceState* device_state(int* code) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        *code = GQA_ERR_DEVICE;
        return nullptr;
    }
    DeviceState& st = g_dev[dev];
    if (!st.checked) {
        st.checked = true;
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) == cudaSuccess && prop.major == 10 && prop.minor == 0) {
            st.num_sms = prop.multiProcessorCount;
            void* sym = nullptr;
            if (cudaGetSymbolAddress(&sym, g_dev_err) == cudaSuccess) {
                st.err = static_cast<int*>(sym);
                st.supported = true;
            }
        }
    }
    if (!st.supported) {
        *code = GQA_ERR_DEVICE;
        return nullptr;
    }
    *code = GQA_OK;
    return &st;
}

// Grow-only workspace.  A grow synchronises the stream first so that no queued kernel still
// uses the old buffer.
bool ensure(void*& ptr, size_t& have, size_t need) {
    if (have >= need) return true;
    if (ptr) {
        cudaStreamSynchronize(g_stream);
        cudaFree(ptr);
        ptr = nullptr;
        have = 0;
    }
    need = (need + 255) & ~size_t(255);
    if (cudaMalloc(&ptr, need) != cudaSuccess) {
        cudaGetLastError();
        ptr = nullptr;
        return false;
    }
    have = need;
    return true;
}

bool get_encoder() {
    if (g_encode) return true;
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
        return false;
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    return true;
}

// bf16 tensor map: innermost dimension d, box {64, ..., 128 rows, ...}, 128-byte swizzle.
bool encode_bf16(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
                 const cuuint32_t* box) {
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides,
                                box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_common(int h_q, int h_kv, int d, float theta) {
    if (h_q <= 0 || h_kv <= 0 || h_q % h_kv != 0) return GQA_ERR_DIMS;
    if (d != 64 && d != 128) return GQA_ERR_HEAD_DIM;
    if (!(theta > 0.0f) || !std::isfinite(theta)) return GQA_ERR_THETA;
    return GQA_OK;
}

// The four tensor maps of the attention kernel: Q' and K' (3-D, rotated workspace), V and out (4-D, the
// caller's tensors in place).
template <int D>
int encode_prefill_maps(CUtensorMap* maps, const void* qr, const void* kr, const void* v, void* out, int B, int L,
                        int h_q, int h_kv) {
    using namespace gqa::prefill;
    if (!get_encoder()) return GQA_ERR_LAUNCH;
    CUtensorMap &tm_q = maps[0], &tm_k = maps[1], &tm_v = maps[2], &tm_o = maps[3];
    const cuuint32_t box3[3] = {64, BM, 1};
    {   // Q' [B*h_q, L, D]
        const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(L),
                                    static_cast<cuuint64_t>(B) * h_q};
        const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(L) * D * 2};
        if (!encode_bf16(&tm_q, const_cast<void*>(qr), 3, dims, strides, box3)) return GQA_ERR_LAUNCH;
    }
    {   // K' [B*h_kv, L, D]
        const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(L),
                                    static_cast<cuuint64_t>(B) * h_kv};
        const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(L) * D * 2};
        if (!encode_bf16(&tm_k, const_cast<void*>(kr), 3, dims, strides, box3)) return GQA_ERR_LAUNCH;
    }
    const cuuint32_t box4[4] = {64, 1, BN, 1};
    {   // V [B, L, h_kv, D], read in place
        const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(h_kv),
                                    static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(B)};
        const cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(h_kv) * D * 2,
                                       static_cast<cuuint64_t>(L) * h_kv * D * 2};
        if (!encode_bf16(&tm_v, v, 4, dims, strides, box4)) return GQA_ERR_LAUNCH;
    }
    {   // out [B, L, h_q, D], written by TMA stores
        const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(h_q),
                                    static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(B)};
        const cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(h_q) * D * 2,
                                       static_cast<cuuint64_t>(L) * h_q * D * 2};
        const cuuint32_t box_o[4] = {64, 1, 32, 1};   // one softmax warp's 32 rows, 64 columns
        if (!encode_bf16(&tm_o, out, 4, dims, strides, box_o)) return GQA_ERR_LAUNCH;
    }

    return GQA_OK;
}

// Per-item overhead of the attention kernel in key tiles, for the schedule below: the start of a pair
// (its query tiles' loads and first scores) and its epilogue.  Measured: with 0 the packing gives some
// CTAs many small items and the kernel is 19 % slower than round-robin at L=4096; 2, 4 and 8 are 3 %,
// 4 % and 2 % faster; against 4, 3 is 4 % slower and 5 the same.
#ifndef GQA_SCHED_ITEM_COST
#define GQA_SCHED_ITEM_COST 4
#endif

// KV planes dealt together when there are many items per CTA, sized for d = 128 whatever d is (the
// schedule is planned without d).  Where the K' and V of all planes fit in well under half of the 126 MB L2
// (48 MB), all of them (no grouping: measured, grouping then only loses the round-robin's order, 3 % at
// B=2, L=8192); otherwise as many as keep 16 MB of K' and V, at least one.  Measured against all planes at
// once on B=4, L=8192 with 64/8 heads (32 planes of 4 MB): groups of 16 MB 8 % fewer cycles per launch,
// of 32 or 64 MB 1-3 %; at L=32768 (4 planes of 16.8 MB, one at a time) 1 %.
#ifndef GQA_GROUP_KV_BYTES
#define GQA_GROUP_KV_BYTES (16ll << 20)
#endif
#ifndef GQA_GROUP_ALL_KV_BYTES
#define GQA_GROUP_ALL_KV_BYTES (48ll << 20)
#endif
int attention_group_planes(int B, int L, int h_kv) {
    const long long per_plane = 2LL * L * 128 * 2;   // K' and V of one (b, u) plane at d = 128
    const long long planes = static_cast<long long>(B) * h_kv;
    if (planes * per_plane <= GQA_GROUP_ALL_KV_BYTES) return static_cast<int>(planes);
    long long g = GQA_GROUP_KV_BYTES / (per_plane > 0 ? per_plane : 1);
    if (g < 1) g = 1;
    if (g > planes) g = planes;
    return static_cast<int>(g);
}

// The attention kernel's work schedule: which items (pairs of query tiles, numbered as in the kernel's
// pair_work) each persistent CTA processes, in order.  Item w costs the key tiles of its two query tiles
// plus a fixed overhead.  With few items per CTA (Qwen2-7B, L=4096: 448 items over 148 CTAs) the balance
// is what matters: the items are dealt heaviest first, each to the fullest CTA that still has room below
// a capacity (best fit decreasing), the capacity raised from its lower bound -- the mean load or the
// largest item -- until everything fits; a round-robin (snake) order would leave the busiest CTA with 9 %
// more work than the average.  With many items per CTA (where that snake order is already within 2 % of
// the packing) any dealing balances: the snake order itself where every plane's K' and V fit L2, else the
// items are dealt for L2 reuse, plane group by plane group (*grouped).  Built on the host once per shape and
// kept on the device (CSR: starts[grid + 1], items).
// Pure host computation of that schedule for B batch rows, L positions, h_q / h_kv heads and `grid` CTAs:
// fills csr (starts[grid + 1], then the items) and returns true for the plane-grouped dealing.
bool plan_attention_schedule(int B, int L, int h_q, int h_kv, int grid, std::vector<int>& csr) {
    constexpr int BM = gqa::prefill::BM;
    const int n_qtiles = (L + BM - 1) / BM, g = h_q / h_kv;
    const int tiles_per_group = n_qtiles * g;
    const int total = (tiles_per_group + 1) / 2 * B * h_kv;   // items, numbered as in the kernel's pair_work
    const int BH = B * h_kv;
    std::vector<long long> cost(total);
    for (int w = 0; w < total; ++w) {
        const int pair = w / BH;
        const int i0 = 2 * pair, i1 = 2 * pair + 1;
        const int n0 = i0 < tiles_per_group ? n_qtiles - i0 / g : 0;
        const int n1 = i1 < tiles_per_group ? n_qtiles - i1 / g : 0;
        cost[w] = n0 + n1 + GQA_SCHED_ITEM_COST;
    }
    // The busiest CTA under the snake order (work_item without a schedule).
    std::vector<long long> snake(grid, 0);
    for (int w = 0; w < total; ++w) {
        const int r = w / grid, c = w % grid;
        snake[(r & 1) ? grid - 1 - c : c] += cost[w];
    }
    const long long snake_max = total > 0 ? *std::max_element(snake.begin(), snake.end()) : 0;
    std::vector<int> order(total);
    std::iota(order.begin(), order.end(), 0);
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return cost[a] > cost[b]; });
    const long long sum = std::accumulate(cost.begin(), cost.end(), 0LL);
    long long cap = std::max((sum + grid - 1) / grid, total > 0 ? cost[order[0]] : 0LL);
    std::vector<std::vector<int>> lists;
    for (;;) {
        lists.assign(grid, {});
        std::set<std::pair<long long, int>> bins;   // (load, cta)
        for (int c = 0; c < grid; ++c) bins.insert({0, c});
        bool fits = true;
        for (int w : order) {
            auto it = bins.upper_bound({cap - cost[w], grid});   // first bin too full for w
            if (it == bins.begin()) {
                fits = false;
                break;
            }
            --it;   // the fullest bin with room
            const auto [load, c] = *it;
            bins.erase(it);
            bins.insert({load + cost[w], c});
            lists[c].push_back(w);
        }
        if (fits) break;
        cap += std::max(1LL, cap / 256);
    }
    const bool many = 100 * snake_max <= 102 * cap;
    const int gp = attention_group_planes(B, L, h_kv);
    if (many && gp >= BH) {
        // Many items per CTA and every plane's K' and V fit L2 together: the round-robin order, every other
        // round reversed (snake), as lists.
        lists.assign(grid, {});
        for (int w = 0; w < total; ++w) {
            const int r = w / grid, c = w % grid;
            lists[(r & 1) ? grid - 1 - c : c].push_back(w);
        }
    } else if (many) {
        // Many items per CTA: any dealing balances, so deal for L2 reuse instead.  The planes (b, u) are
        // taken a group at a time (attention_group_planes), each group's items heaviest first to the least
        // loaded CTA: every CTA runs through the groups in the same order, so the K' and V tiles read at
        // any moment belong to one group or two and stay in L2.  With all planes at once the B=4, L=8192,
        // 64/8-head workload read its K' and V from DRAM about six times over.
        const int pairs = total / BH;
        lists.assign(grid, {});
        std::set<std::pair<long long, int>> bins;   // (load, cta)
        for (int c = 0; c < grid; ++c) bins.insert({0, c});
        std::vector<int> grp_items;
        for (int g0 = 0; g0 < BH; g0 += gp) {
            grp_items.clear();
            for (int pr = 0; pr < pairs; ++pr)
                for (int pl = g0; pl < std::min(BH, g0 + gp); ++pl) grp_items.push_back(pr * BH + pl);
            std::stable_sort(grp_items.begin(), grp_items.end(), [&](int a, int b) { return cost[a] > cost[b]; });
            for (int w : grp_items) {
                auto it = bins.begin();   // the least loaded CTA
                const auto [load, c] = *it;
                bins.erase(it);
                bins.insert({load + cost[w], c});
                lists[c].push_back(w);
            }
        }
    }
    csr.assign(static_cast<size_t>(grid) + 1 + total, 0);
    int at = 0;
    for (int c = 0; c < grid; ++c) {
        csr[c] = at;
        for (int w : lists[c]) csr[grid + 1 + at++] = w;
    }
    csr[grid] = at;
    return many && gp < BH;
}

int attention_schedule(DeviceState* st, const gqa::prefill::Params& p, int grid) {
    const int key[5] = {p.B, p.L, p.h_q, p.h_kv, grid};
    if (st->sched_valid && std::equal(key, key + 5, st->sched_key)) return GQA_OK;
    st->sched_valid = false;
    std::vector<int> csr;
    plan_attention_schedule(p.B, p.L, p.h_q, p.h_kv, grid, csr);
    std::copy(key, key + 5, st->sched_key);
    st->sched_valid = true;
    const size_t bytes = csr.size() * sizeof(int);
    if (!ensure(st->sched, st->sched_bytes, bytes)) {
        st->sched_valid = false;
        return GQA_ERR_ALLOC;
    }
    // Pageable source: the copy has read it when the call returns; ordered before the kernel on the stream.
    if (cudaMemcpyAsync(st->sched, csr.data(), bytes, cudaMemcpyHostToDevice, g_stream) != cudaSuccess) {
        st->sched_valid = false;
        return GQA_ERR_LAUNCH;
    }
    return GQA_OK;
}

// The attention kernel over rotated Q' [B, h_q, L, D], K' [B, h_kv, L, D] and V [B, L, h_kv, D].  A plain
// launch after the kernel that writes Q' and K': as a programmatic dependent of the prep kernel (CTAs
// placed while the prep grid drains, then waiting for it) the attention measured 1-4 % slower per step.
template <int D>
int launch_attention(DeviceState* st, const void* qr, const void* kr, const void* v, void* out, int B, int L,
                     int h_q, int h_kv) {
    using namespace gqa::prefill;
    const DeviceState::MapKey key{qr, kr, v, out, B, L, h_q, h_kv, D};
    if (!st->maps_valid || !(st->map_key == key)) {
        st->maps_valid = false;
        const int rc = encode_prefill_maps<D>(st->maps, qr, kr, v, out, B, L, h_q, h_kv);
        if (rc != GQA_OK) return rc;
        st->map_key = key;
        st->maps_valid = true;
    }

    Params p;
    p.out = static_cast<__nv_bfloat16*>(out);
    p.B = B;
    p.L = L;
    p.h_q = h_q;
    p.h_kv = h_kv;
    p.g = h_q / h_kv;
    p.n_qtiles = (L + BM - 1) / BM;
    p.tiles_per_group = p.n_qtiles * p.g;
    p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
    p.err = st->err;
    const long long total = static_cast<long long>((p.tiles_per_group + 1) / 2) * B * h_kv;
    if (total > 0x7fffffffLL) return GQA_ERR_DIMS;
    p.total_work = static_cast<int>(total);
    // Persistent: one CTA per SM (each holds a whole SM's tensor memory), at most one per work item.
    const int grid = static_cast<int>(total < st->num_sms ? total : st->num_sms);
    const int rc = attention_schedule(st, p, grid);
    if (rc != GQA_OK) return rc;
    p.sched_start = static_cast<const int*>(st->sched);
    p.sched = static_cast<const int*>(st->sched) + grid + 1;
    bool& ready = st->attn_ready[D == 128 ? 1 : 0];
    if (!ready) {
        if (cudaFuncSetAttribute(attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, Layout<D>::DYN) !=
            cudaSuccess)
            return GQA_ERR_LAUNCH;
        // The in-kernel register split (setmaxnreg) is only valid for this exact launch budget.
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, attn_kernel<D>) != cudaSuccess || fa.numRegs != LAUNCH_REGS)
            return GQA_ERR_LAUNCH;
        ready = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(NUM_THREADS);
    cfg.dynamicSmemBytes = Layout<D>::DYN;
    cfg.stream = g_stream;
    mark(g_ev_start);
    if (cudaLaunchKernelEx(&cfg, attn_kernel<D>, st->maps[0], st->maps[1], st->maps[2], st->maps[3], p) !=
        cudaSuccess)
        return GQA_ERR_LAUNCH;
    mark(g_ev_stop);
    return GQA_OK;
}

template <int D>
int launch_prefill(DeviceState* st, const void* q, const void* k, const void* v, void* out, int B, int L, int h_q,
                   int h_kv, float theta) {
    using namespace gqa::prefill;
    // Workspace: Q' [B*h_q, L, D] then K' [B*h_kv, L, D], both bf16, rotated.
    const size_t qr_bytes = (static_cast<size_t>(B) * h_q * L * D * 2 + 255) & ~size_t(255);
    const size_t kr_bytes = static_cast<size_t>(B) * h_kv * L * D * 2;
    if (!ensure(st->ws, st->ws_bytes, qr_bytes + kr_bytes)) return GQA_ERR_ALLOC;
    auto* qr = static_cast<__nv_bfloat16*>(st->ws);
    auto* kr = reinterpret_cast<__nv_bfloat16*>(static_cast<uint8_t*>(st->ws) + qr_bytes);

    const int prep_blocks = (L + PREP_POS - 1) / PREP_POS;
    prep_kernel<D><<<prep_blocks, PREP_THREADS, 0, g_stream>>>(static_cast<const __nv_bfloat16*>(q),
                                                               static_cast<const __nv_bfloat16*>(k), qr, kr, B, L,
                                                               h_q, h_kv, rope_spec(theta), rope_mscale());
    if (cudaGetLastError() != cudaSuccess) return GQA_ERR_LAUNCH;
    return launch_attention<D>(st, qr, kr, v, out, B, L, h_q, h_kv);
}

// The cos / sin table for positions 0 .. L-1, rebuilt only when (L, d, theta) changes.
template <int D>
int ensure_rope_table(DeviceState* st, int L, float theta) {
    using namespace gqa::qkv;
    if (st->tab && st->tab_L >= L && st->tab_d == D && st->tab_theta == theta && st->tab_factor == g_rope_factor &&
        st->tab_orig == g_rope_orig)
        return GQA_OK;
    const size_t bytes = static_cast<size_t>(L) * (D / 2) * sizeof(float2);
    if (!ensure(st->tab, st->tab_bytes, bytes)) return GQA_ERR_ALLOC;
    const long long n = static_cast<long long>(L) * (D / 2);
    rope_table_kernel<D><<<static_cast<unsigned>((n + TABLE_THREADS - 1) / TABLE_THREADS), TABLE_THREADS, 0,
                           g_stream>>>(static_cast<float2*>(st->tab), L, rope_spec(theta), rope_mscale());
    if (cudaGetLastError() != cudaSuccess) return GQA_ERR_LAUNCH;
    st->tab_L = L;
    st->tab_d = D;
    st->tab_theta = theta;
    st->tab_factor = g_rope_factor;
    st->tab_orig = g_rope_orig;
    return GQA_OK;
}

// X [T, K] and W [N, K] tensor maps of a projection GEMM with tile width bn, and W again with the box of
// a tail unit (TAIL_BN rows); reused while the key matches.
bool gemm_maps(CUtensorMap* maps, const void** key, long long* dims, const void* x, const void* w, long long T,
               int K, long long N, int bn) {
    using namespace gqa::qkv;
    if (key[0] == x && key[1] == w && dims[0] == T && dims[1] == N && dims[2] == K && dims[3] == bn) return true;
    key[0] = key[1] = nullptr;
    if (!get_encoder()) return false;
    const cuuint64_t sx[1] = {static_cast<cuuint64_t>(K) * 2};
    const cuuint64_t dx[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(T)};
    const cuuint32_t bx[2] = {BK, BM};
    if (!encode_bf16(&maps[0], const_cast<void*>(x), 2, dx, sx, bx)) return false;
    const cuuint64_t dw[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(N)};
    const cuuint32_t bw[2] = {BK, static_cast<cuuint32_t>(bn)};
    if (!encode_bf16(&maps[1], const_cast<void*>(w), 2, dw, sx, bw)) return false;
    const cuuint32_t bt[2] = {BK, static_cast<cuuint32_t>(TAIL_BN)};
    if (!encode_bf16(&maps[2], const_cast<void*>(w), 2, dw, sx, bt)) return false;
    key[0] = x;
    key[1] = w;
    dims[0] = T;
    dims[1] = N;
    dims[2] = K;
    dims[3] = bn;
    return true;
}

// Launch one instantiation of the persistent GEMM (the kernel `fn`, tile width BN) over p.n_tiles tiles.
// With `split_tail`, a last wave at most a quarter full is split into BN / TAIL_BN-column units, so that
// it occupies four times as many CTAs for a quarter of the time each (the output projection: the
// 4096 x 3584 product is 448 tiles = 3 waves of 148 and 4 tiles).
template <int BN>
int run_gemm(DeviceState* st, void (*fn)(CUtensorMap, CUtensorMap, CUtensorMap, gqa::qkv::Params),
             unsigned ready_bit, const CUtensorMap* maps, gqa::qkv::Params p, bool split_tail) {
    using namespace gqa::qkv;
    if (!(st->gemm_ready & ready_bit)) {
        if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, Tile<BN>::DYN) != cudaSuccess)
            return GQA_ERR_LAUNCH;
        st->gemm_ready |= ready_bit;
    }
    const int grid = p.n_tiles < st->num_sms ? p.n_tiles : st->num_sms;
    const int last = p.n_tiles % grid;   // tiles in a partly filled last wave
    constexpr int SPLIT = BN / TAIL_BN;
    p.n_main = p.n_tiles;
    p.tail_split = 1;
    if (split_tail && SPLIT > 1 && last > 0 && last * SPLIT <= grid) {
        p.n_main = p.n_tiles - last;
        p.tail_split = SPLIT;
    }
    p.n_units = p.n_main + (p.n_tiles - p.n_main) * p.tail_split;
    mark(g_ev_start);
    fn<<<grid, NUM_THREADS, Tile<BN>::DYN, g_stream>>>(maps[0], maps[1], maps[2], p);
    if (cudaGetLastError() != cudaSuccess) return GQA_ERR_LAUNCH;
    mark(g_ev_stop);
    return GQA_OK;
}

template <int D>
int launch_qkv(DeviceState* st, const void* x, const void* w, const void* bias, void* qr, void* kr, void* k,
               void* v, int B, int L, int d_model, int h_q, int h_kv, float theta) {
    using namespace gqa::qkv;
    int rc = ensure_rope_table<D>(st, L, theta);
    if (rc != GQA_OK) return rc;
    const long long T = static_cast<long long>(B) * L;
    const int N = (h_q + 2 * h_kv) * D;
    const long long mtiles = (T + BM - 1) / BM;
    constexpr int bn = 256;
    if (!gemm_maps(st->qkv_maps, st->qkv_key, st->qkv_dims, x, w, T, d_model, N, bn)) return GQA_ERR_LAUNCH;
    Params p = {};
    p.bias = static_cast<const __nv_bfloat16*>(bias);
    p.tab = static_cast<const float2*>(st->tab);
    p.k_rotated = g_cache_rotated;
    p.qr = static_cast<__nv_bfloat16*>(qr);
    p.kr = static_cast<__nv_bfloat16*>(kr);
    p.k = static_cast<__nv_bfloat16*>(k);
    p.v = static_cast<__nv_bfloat16*>(v);
    p.T = static_cast<int>(T);
    p.L = L;
    p.N = N;
    p.h_q = h_q;
    p.h_kv = h_kv;
    p.n_ntiles = (N + bn - 1) / bn;
    if (mtiles * p.n_ntiles > 0x7fffffffLL) return GQA_ERR_DIMS;
    p.n_tiles = static_cast<int>(mtiles * p.n_ntiles);
    p.kblocks = (d_model + BK - 1) / BK;
    p.err = st->err;
    return run_gemm<bn>(st, qkv_kernel<D, bn>, D == 128 ? 1u : 2u, st->qkv_maps, p, false);
}

// Output projection + residual: out [T, d_model] = attn [T, d_in] w_o [d_model, d_in]^T (+ resid).
int launch_proj(DeviceState* st, const void* attn, const void* w_o, const void* resid, void* out, int T, int d_in,
                int d_model) {
    using namespace gqa::qkv;
    const long long mtiles = (static_cast<long long>(T) + BM - 1) / BM;
    constexpr int bn = 256;
    if (!gemm_maps(st->proj_maps, st->proj_key, st->proj_dims, attn, w_o, T, d_in, d_model, bn))
        return GQA_ERR_LAUNCH;
    Params p = {};
    p.resid = static_cast<const __nv_bfloat16*>(resid);
    p.out = static_cast<__nv_bfloat16*>(out);
    p.T = T;
    p.L = T;
    p.N = d_model;
    p.n_ntiles = (d_model + bn - 1) / bn;
    if (mtiles * p.n_ntiles > 0x7fffffffLL) return GQA_ERR_DIMS;
    p.n_tiles = static_cast<int>(mtiles * p.n_ntiles);
    p.kblocks = (d_in + BK - 1) / BK;
    p.err = st->err;
    return run_gemm<bn>(st, proj_kernel<bn>, 4u, st->proj_maps, p, true);
}

// One decode step's projection and cache append: x [B, d_model] (the new token of each sequence) times
// w_qkv^T + bias; q [B, h_q, D] and the page slots of positions seqlens[b] get the un-rotated heads.
template <int D>
int launch_append(DeviceState* st, const void* x, const void* w, const void* bias, const int* seqlens, void* q,
                  void* kpages, void* vpages, const int* bt, int B, int d_model, int h_q, int h_kv, int page_size,
                  int num_pages, int max_pages, float theta) {
    using namespace gqa::qkv;
    const int N = (h_q + 2 * h_kv) * D;
    const long long mtiles = (static_cast<long long>(B) + BM - 1) / BM;
    constexpr int bn = 256;
    if (!gemm_maps(st->app_maps, st->app_key, st->app_dims, x, w, B, d_model, N, bn)) return GQA_ERR_LAUNCH;
    Params p = {};
    p.bias = static_cast<const __nv_bfloat16*>(bias);
    p.qr = static_cast<__nv_bfloat16*>(q);
    p.k = static_cast<__nv_bfloat16*>(kpages);
    p.v = static_cast<__nv_bfloat16*>(vpages);
    p.seqlens = seqlens;
    p.bt = bt;
    p.page_size = page_size;
    p.num_pages = num_pages;
    p.max_pages = max_pages;
    p.k_rotated = g_cache_rotated;
    p.rope = rope_spec(theta);
    p.mscale = rope_mscale();
    p.T = B;
    p.L = 1;
    p.N = N;
    p.h_q = h_q;
    p.h_kv = h_kv;
    p.n_ntiles = (N + bn - 1) / bn;
    if (mtiles * p.n_ntiles > 0x7fffffffLL) return GQA_ERR_DIMS;
    p.n_tiles = static_cast<int>(mtiles * p.n_ntiles);
    p.kblocks = (d_model + BK - 1) / BK;
    p.err = st->err;
    return run_gemm<bn>(st, append_kernel<D, bn>, D == 128 ? 8u : 16u, st->app_maps, p, false);
}

// The decode step's three kernels: plan (offsets), split (one partial per piece), combine (merge).
// Split and combine are programmatic dependents of the kernel before them: their CTAs may start
// (barrier and RoPE-table set-up) while it drains, and wait for its results with griddepcontrol.wait.
// With timing events around the split kernel (`marks` and events set) the launches are plain.
template <int D>
int launch_decode_chain(const gqa::decode::Params& p, const int* seqlens, int64_t* off, int split_grid, bool marks) {
    using namespace gqa::decode;
    using C = Cfg<D>;
    const long long cgrid = static_cast<long long>(p.B) * p.h_kv * p.n_hb;
    if (cgrid > 0x7fffffffLL) return GQA_ERR_DIMS;
    const bool paged = p.bt != nullptr;
    auto split = paged ? (g_cache_rotated ? split_kernel<D, true, true> : split_kernel<D, true, false>)
                       : (g_cache_rotated ? split_kernel<D, false, true> : split_kernel<D, false, false>);
    if (cudaFuncSetAttribute(split, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
        return GQA_ERR_LAUNCH;
    const bool timed = marks && g_ev_start && g_ev_stop;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.stream = g_stream;
    cfg.attrs = attr;
    cfg.numAttrs = 0;
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(PLAN_THREADS);
    if (cudaLaunchKernelEx(&cfg, plan_kernel, seqlens, off, p.B, p.err) != cudaSuccess) return GQA_ERR_LAUNCH;
    if (marks) mark(g_ev_start);
    cfg.numAttrs = timed ? 0 : 1;
    cfg.gridDim = dim3(split_grid);
    cfg.blockDim = dim3(WARPS * 32);
    cfg.dynamicSmemBytes = C::SMEM;
    if (cudaLaunchKernelEx(&cfg, split, p) != cudaSuccess) return GQA_ERR_LAUNCH;
    if (marks) mark(g_ev_stop);
    cfg.gridDim = dim3(static_cast<unsigned>(cgrid));
    cfg.blockDim = dim3(COMBINE_THREADS);
    cfg.dynamicSmemBytes = 0;
    if (cudaLaunchKernelEx(&cfg, combine_kernel<D>, p) != cudaSuccess) return GQA_ERR_LAUNCH;
    return GQA_OK;
}

// Packed cache (bt == nullptr) or paged cache through the block table bt [B, max_pages].
template <int D>
int launch_decode(DeviceState* st, const void* q, const void* kc, const void* vc, const int* seqlens, void* out,
                  int B, int h_q, int h_kv, float theta, const int* bt = nullptr, int page_size = 0,
                  int num_pages = 0, int max_pages = 0) {
    using namespace gqa::decode;
    using C = Cfg<D>;
    const int g = h_q / h_kv;
    const int n_hb = (g + HB - 1) / HB;
    const int groups = h_kv * n_hb;
    // CTAS_PER_SM CTAs of WARPS workers per SM in total, split evenly over the (group, head block) pairs.
    const int G = (CTAS_PER_SM * st->num_sms + groups - 1) / groups;
    const int P = G * WARPS;
    const size_t off_bytes = ((static_cast<size_t>(B) + 1) * sizeof(int64_t) + 255) & ~size_t(255);
    const size_t part_bytes = (static_cast<size_t>(P) + static_cast<size_t>(B)) * groups * C::PART * sizeof(float);
    if (!ensure(st->dws, st->dws_bytes, off_bytes + part_bytes)) return GQA_ERR_ALLOC;

    Params p;
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.kc = static_cast<const __nv_bfloat16*>(kc);
    p.vc = static_cast<const __nv_bfloat16*>(vc);
    p.out = static_cast<__nv_bfloat16*>(out);
    p.bt = bt;
    p.page_size = page_size;
    p.num_pages = num_pages;
    p.max_pages = max_pages;
    p.off = static_cast<int64_t*>(st->dws);
    p.part = reinterpret_cast<float*>(static_cast<uint8_t*>(st->dws) + off_bytes);
    p.B = B;
    p.h_q = h_q;
    p.h_kv = h_kv;
    p.g = g;
    p.n_hb = n_hb;
    p.P = P;
    p.self_in_cache = g_self_in_cache;
    p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
    p.rope = rope_spec(theta);
    // YaRN temperature on q and on each key (1 without scaling); a rotated cache's keys already carry theirs.
    p.scale_log2 *= rope_mscale() * (g_cache_rotated ? 1.0f : rope_mscale());
    p.err = st->err;

    return launch_decode_chain<D>(p, seqlens, static_cast<int64_t*>(st->dws), G * groups, true);
}

// ---------------------------------------------------------------------------------------------
// Decode without any device allocation (gqa_decode_noalloc).
//
// Who needs it: callers that own every byte of device memory themselves -- for example a serving
// process that reserves almost all of HBM for its KV cache and model at start-up, where a cudaMalloc
// from inside a library would fail or fragment that reservation -- and callers on a latency-critical
// path that cannot pay for cudaMalloc / cudaFree, which may synchronise the whole device.  For them the
// decode scratch (packed row offsets and split partials) lives in this fixed, file-scope device array,
// which every GPU that loads the library holds until the process exits.
constexpr size_t kFixedScratchBytes = size_t(16) << 20;   // 16 MiB per device
static __device__ __align__(256) unsigned char g_fixed_scratch[kFixedScratchBytes];

// In host code `g_fixed_scratch` names a host-side stand-in, not device memory: kernels must be given
// the device address, looked up once per device with that device current.
int fixed_scratch_setup(DeviceState* st) {
    if (st->fixed_scratch) return GQA_OK;
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_fixed_scratch) != cudaSuccess || ptr == nullptr) {
        cudaGetLastError();
        return GQA_ERR_LAUNCH;
    }
    st->fixed_scratch = ptr;
    return GQA_OK;
}

template <int D>
int launch_decode_fixed_scratch(DeviceState* st, const void* q, const void* kc, const void* vc, const int* seqlens,
                                void* out, int B, int h_q, int h_kv, float theta) {
    using namespace gqa::decode;
    using C = Cfg<D>;
    const int g = h_q / h_kv;
    const int n_hb = (g + HB - 1) / HB;
    const int groups = h_kv * n_hb;
    const int G = (CTAS_PER_SM * st->num_sms + groups - 1) / groups;
    const int P = G * WARPS;
    const size_t off_bytes = ((static_cast<size_t>(B) + 1) * sizeof(int64_t) + 255) & ~size_t(255);
    const size_t part_bytes = (static_cast<size_t>(P) + static_cast<size_t>(B)) * groups * C::PART * sizeof(float);
    if (off_bytes + part_bytes > kFixedScratchBytes) return GQA_ERR_TOO_LARGE;
    const int rc = fixed_scratch_setup(st);
    if (rc != GQA_OK) return rc;

    // Nothing in the scratch has to start at zero: plan_kernel rewrites all B + 1 offsets, and the
    // combine step reads only the partials that split_kernel wrote in this same call.
    Params p;
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.kc = static_cast<const __nv_bfloat16*>(kc);
    p.vc = static_cast<const __nv_bfloat16*>(vc);
    p.out = static_cast<__nv_bfloat16*>(out);
    p.bt = nullptr;
    p.page_size = p.num_pages = p.max_pages = 0;
    p.off = static_cast<int64_t*>(st->fixed_scratch);
    p.part = reinterpret_cast<float*>(static_cast<uint8_t*>(st->fixed_scratch) + off_bytes);
    p.B = B;
    p.h_q = h_q;
    p.h_kv = h_kv;
    p.g = g;
    p.n_hb = n_hb;
    p.P = P;
    p.self_in_cache = g_self_in_cache;
    p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
    p.rope = rope_spec(theta);
    // YaRN temperature on q and on each key (1 without scaling); a rotated cache's keys already carry theirs.
    p.scale_log2 *= rope_mscale() * (g_cache_rotated ? 1.0f : rope_mscale());
    p.err = st->err;

    return launch_decode_chain<D>(p, seqlens, static_cast<int64_t*>(st->fixed_scratch), G * groups, false);
}

}  // namespace

extern "C" {

int gqa_abi_version(void) { return 2; }

const char* gqa_strerror(int code) {
    switch (code) {
        case GQA_OK: return "success";
        case GQA_ERR_NULL: return "a required pointer is NULL";
        case GQA_ERR_DIMS: return "invalid sizes (negative, h_q not a multiple of h_kv, or too large)";
        case GQA_ERR_HEAD_DIM: return "unsupported head dimension (must be 64 or 128)";
        case GQA_ERR_THETA: return "RoPE base theta must be positive and finite";
        case GQA_ERR_LAUNCH: return "CUDA launch or tensor-map encoding failed";
        case GQA_ERR_ALLOC: return "workspace allocation failed";
        case GQA_ERR_ALIGN: return "a tensor pointer is not 16-byte aligned";
        case GQA_ERR_DEVICE: return "the current CUDA device is not an sm_100 GPU";
        case GQA_ERR_TOO_LARGE: return "the decode needs more scratch than the fixed 16 MiB buffer of gqa_decode_noalloc";
        default: return "unknown error code";
    }
}

int gqa_set_timing_events(void* start_event, void* stop_event) {
    g_ev_start = static_cast<cudaEvent_t>(start_event);
    g_ev_stop = static_cast<cudaEvent_t>(stop_event);
    return GQA_OK;
}

int gqa_set_rope_scaling(float factor, int original_max_position) {
    if (!(factor >= 1.0f) || !std::isfinite(factor)) return GQA_ERR_DIMS;
    if (factor > 1.0f && original_max_position <= 0) return GQA_ERR_DIMS;
    g_rope_factor = factor;
    g_rope_orig = factor > 1.0f ? original_max_position : 0;
    return GQA_OK;
}

int gqa_set_stream(void* cuda_stream) {
    g_stream = static_cast<cudaStream_t>(cuda_stream);
    return GQA_OK;
}

int gqa_prefill(const void* q, const void* k, const void* v, void* out, int B, int L, int h_q, int h_kv, int d,
                float theta) {
    if (B < 0 || L < 0) return GQA_ERR_DIMS;
    int rc = check_common(h_q, h_kv, d, theta);
    if (rc != GQA_OK) return rc;
    if (B == 0 || L == 0) return GQA_OK;
    if (!q || !k || !v || !out) return GQA_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return GQA_ERR_ALIGN;
    // TMA coordinates are 32-bit and the kernel indexes rows with 32-bit positions.
    // TMA coordinates are 32-bit; the prep kernel indexes B * (h_q + h_kv) * 8 * d / 16 items in 32 bits.
    if (static_cast<long long>(B) * (h_q + h_kv) * 64 > 0x7fffffffLL || L > (1 << 30)) return GQA_ERR_DIMS;
    DeviceState* st = device_state(&rc);
    if (!st) return rc;
    return d == 64 ? launch_prefill<64>(st, q, k, v, out, B, L, h_q, h_kv, theta)
                   : launch_prefill<128>(st, q, k, v, out, B, L, h_q, h_kv, theta);
}

int gqa_decode(const void* q, const void* kcache, const void* vcache, const int* seqlens, void* out, int B, int h_q,
               int h_kv, int d, float theta) {
    if (B < 0) return GQA_ERR_DIMS;
    int rc = check_common(h_q, h_kv, d, theta);
    if (rc != GQA_OK) return rc;
    if (B == 0) return GQA_OK;
    if (!q || !kcache || !vcache || !seqlens || !out) return GQA_ERR_NULL;
    if (!aligned16(q) || !aligned16(kcache) || !aligned16(vcache) || !aligned16(out)) return GQA_ERR_ALIGN;
    DeviceState* st = device_state(&rc);
    if (!st) return rc;
    return d == 64 ? launch_decode<64>(st, q, kcache, vcache, seqlens, out, B, h_q, h_kv, theta)
                   : launch_decode<128>(st, q, kcache, vcache, seqlens, out, B, h_q, h_kv, theta);
}

int gqa_decode_noalloc(const void* q, const void* kcache, const void* vcache, const int* seqlens, void* out, int B,
                       int h_q, int h_kv, int d, float theta) {
    if (B < 0) return GQA_ERR_DIMS;
    int rc = check_common(h_q, h_kv, d, theta);
    if (rc != GQA_OK) return rc;
    if (B == 0) return GQA_OK;
    if (!q || !kcache || !vcache || !seqlens || !out) return GQA_ERR_NULL;
    if (!aligned16(q) || !aligned16(kcache) || !aligned16(vcache) || !aligned16(out)) return GQA_ERR_ALIGN;
    DeviceState* st = device_state(&rc);
    if (!st) return rc;
    return d == 64 ? launch_decode_fixed_scratch<64>(st, q, kcache, vcache, seqlens, out, B, h_q, h_kv, theta)
                   : launch_decode_fixed_scratch<128>(st, q, kcache, vcache, seqlens, out, B, h_q, h_kv, theta);
}

int gqa_decode_paged(const void* q, const void* kpages, const void* vpages, const int* block_table,
                     const int* seqlens, void* out, int B, int h_q, int h_kv, int d, int page_size, int num_pages,
                     int max_pages_per_seq, float theta) {
    if (B < 0 || page_size <= 0 || num_pages <= 0 || max_pages_per_seq <= 0) return GQA_ERR_DIMS;
    // Storage rows are indexed page * page_size + slot in 64 bits; positions stay below 2^31.
    if (static_cast<long long>(num_pages) * page_size > (1LL << 40)) return GQA_ERR_DIMS;
    if (static_cast<long long>(B) * max_pages_per_seq > 0x7fffffffLL) return GQA_ERR_DIMS;
    int rc = check_common(h_q, h_kv, d, theta);
    if (rc != GQA_OK) return rc;
    if (B == 0) return GQA_OK;
    if (!q || !kpages || !vpages || !block_table || !seqlens || !out) return GQA_ERR_NULL;
    if (!aligned16(q) || !aligned16(kpages) || !aligned16(vpages) || !aligned16(out)) return GQA_ERR_ALIGN;
    DeviceState* st = device_state(&rc);
    if (!st) return rc;
    return d == 64 ? launch_decode<64>(st, q, kpages, vpages, seqlens, out, B, h_q, h_kv, theta, block_table,
                                       page_size, num_pages, max_pages_per_seq)
                   : launch_decode<128>(st, q, kpages, vpages, seqlens, out, B, h_q, h_kv, theta, block_table,
                                        page_size, num_pages, max_pages_per_seq);
}

int gqa_qkv_rope(const void* x, const void* w_qkv, const void* b_qkv, void* qr, void* kr, void* k, void* v, int B,
                 int L, int d_model, int h_q, int h_kv, int d, float theta) {
    if (B < 0 || L < 0 || d_model <= 0 || d_model % 8 != 0) return GQA_ERR_DIMS;
    int rc = check_common(h_q, h_kv, d, theta);
    if (rc != GQA_OK) return rc;
    if (B == 0 || L == 0) return GQA_OK;
    if (!x || !w_qkv || !qr || !kr || !k || !v) return GQA_ERR_NULL;
    if (!aligned16(x) || !aligned16(w_qkv) || !aligned16(qr) || !aligned16(kr) || !aligned16(k) || !aligned16(v) ||
        (b_qkv && !aligned16(b_qkv)))
        return GQA_ERR_ALIGN;
    // Token rows and output columns are TMA coordinates (32-bit); positions stay below 2^30.
    if (static_cast<long long>(B) * L > 0x7fffffffLL || L > (1 << 30) ||
        static_cast<long long>(h_q + 2 * h_kv) * d > 0x7fffffffLL)
        return GQA_ERR_DIMS;
    DeviceState* st = device_state(&rc);
    if (!st) return rc;
    return d == 64 ? launch_qkv<64>(st, x, w_qkv, b_qkv, qr, kr, k, v, B, L, d_model, h_q, h_kv, theta)
                   : launch_qkv<128>(st, x, w_qkv, b_qkv, qr, kr, k, v, B, L, d_model, h_q, h_kv, theta);
}

int gqa_qkv_append(const void* x, const void* w_qkv, const void* b_qkv, const int* seqlens, void* q, void* kpages,
                   void* vpages, const int* block_table, int B, int d_model, int h_q, int h_kv, int d, int page_size,
                   int num_pages, int max_pages_per_seq, float theta) {
    if (B < 0 || d_model <= 0 || d_model % 8 != 0 || page_size <= 0 || num_pages <= 0 || max_pages_per_seq <= 0)
        return GQA_ERR_DIMS;
    if (static_cast<long long>(num_pages) * page_size > (1LL << 40)) return GQA_ERR_DIMS;
    if (static_cast<long long>(B) * max_pages_per_seq > 0x7fffffffLL) return GQA_ERR_DIMS;
    int rc = check_common(h_q, h_kv, d, theta);
    if (rc != GQA_OK) return rc;
    if (B == 0) return GQA_OK;
    if (!x || !w_qkv || !seqlens || !q || !kpages || !vpages || !block_table) return GQA_ERR_NULL;
    if (!aligned16(x) || !aligned16(w_qkv) || !aligned16(q) || !aligned16(kpages) || !aligned16(vpages) ||
        (b_qkv && !aligned16(b_qkv)))
        return GQA_ERR_ALIGN;
    if (static_cast<long long>(h_q + 2 * h_kv) * d > 0x7fffffffLL) return GQA_ERR_DIMS;
    DeviceState* st = device_state(&rc);
    if (!st) return rc;
    return d == 64 ? launch_append<64>(st, x, w_qkv, b_qkv, seqlens, q, kpages, vpages, block_table, B, d_model, h_q,
                                       h_kv, page_size, num_pages, max_pages_per_seq, theta)
                   : launch_append<128>(st, x, w_qkv, b_qkv, seqlens, q, kpages, vpages, block_table, B, d_model,
                                        h_q, h_kv, page_size, num_pages, max_pages_per_seq, theta);
}

int gqa_set_decode_self_in_cache(int on) {
    if (on != 0 && on != 1) return GQA_ERR_DIMS;
    g_self_in_cache = on;
    return GQA_OK;
}

int gqa_set_decode_cache_rotated(int on) {
    if (on != 0 && on != 1) return GQA_ERR_DIMS;
    g_cache_rotated = on;
    return GQA_OK;
}

int gqa_out_proj(const void* attn, const void* w_o, const void* residual, void* out, int T, int d_in, int d_model) {
    if (T < 0 || d_in <= 0 || d_in % 8 != 0 || d_model <= 0 || d_model % 128 != 0) return GQA_ERR_DIMS;
    if (T == 0) return GQA_OK;
    if (!attn || !w_o || !out) return GQA_ERR_NULL;
    if (!aligned16(attn) || !aligned16(w_o) || !aligned16(out) || (residual && !aligned16(residual)))
        return GQA_ERR_ALIGN;
    int rc = GQA_OK;
    DeviceState* st = device_state(&rc);
    if (!st) return rc;
    return launch_proj(st, attn, w_o, residual, out, T, d_in, d_model);
}

int gqa_prefill_rotated(const void* qr, const void* kr, const void* v, void* out, int B, int L, int h_q, int h_kv,
                        int d) {
    if (B < 0 || L < 0) return GQA_ERR_DIMS;
    int rc = check_common(h_q, h_kv, d, 1.0f);
    if (rc != GQA_OK) return rc;
    if (B == 0 || L == 0) return GQA_OK;
    if (!qr || !kr || !v || !out) return GQA_ERR_NULL;
    if (!aligned16(qr) || !aligned16(kr) || !aligned16(v) || !aligned16(out)) return GQA_ERR_ALIGN;
    if (static_cast<long long>(B) * (h_q + h_kv) * 64 > 0x7fffffffLL || L > (1 << 30)) return GQA_ERR_DIMS;
    DeviceState* st = device_state(&rc);
    if (!st) return rc;
    return d == 64 ? launch_attention<64>(st, qr, kr, v, out, B, L, h_q, h_kv)
                   : launch_attention<128>(st, qr, kr, v, out, B, L, h_q, h_kv);
}

int gqa_last_error(void) {
    int rc = GQA_OK;
    DeviceState* st = device_state(&rc);
    if (!st) return rc;
    if (cudaStreamSynchronize(g_stream) != cudaSuccess) return GQA_ERR_LAUNCH;
    int h = 0;
    if (cudaMemcpyFromSymbol(&h, g_dev_err, sizeof(int)) != cudaSuccess) return GQA_ERR_LAUNCH;
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_dev_err, &zero, sizeof(int)) != cudaSuccess) return GQA_ERR_LAUNCH;
    return h;
}

int gqa_prefill_schedule(int B, int L, int h_q, int h_kv, int grid, int* starts, int* items, int capacity,
                         int* grouped) {
    if (B <= 0 || L <= 0 || h_q <= 0 || h_kv <= 0 || h_q % h_kv != 0 || grid <= 0) return GQA_ERR_DIMS;
    const long long total = static_cast<long long>((L + 127) / 128 * (h_q / h_kv) + 1) / 2 * B * h_kv;
    if (total > 0x7fffffffLL || static_cast<long long>(B) * (h_q + h_kv) * 64 > 0x7fffffffLL || L > (1 << 30))
        return GQA_ERR_DIMS;
    const int g = total < grid ? static_cast<int>(total) : grid;
    std::vector<int> csr;
    const bool by_group = plan_attention_schedule(B, L, h_q, h_kv, g, csr);
    if (grouped) *grouped = by_group ? 1 : 0;
    if (starts && items && capacity >= total) {
        std::copy(csr.begin(), csr.begin() + g + 1, starts);
        std::copy(csr.begin() + g + 1, csr.end(), items);
    }
    return static_cast<int>(total);
}

void gqa_release(void) {
    int cur = 0;
    if (cudaGetDevice(&cur) != cudaSuccess) return;
    for (int dev = 0; dev < kMaxDevices; ++dev) {
        DeviceState& st = g_dev[dev];
        if (!st.ws && !st.dws && !st.tab && !st.sched) continue;
        cudaSetDevice(dev);
        cudaDeviceSynchronize();
        if (st.ws) cudaFree(st.ws);
        if (st.dws) cudaFree(st.dws);
        if (st.tab) cudaFree(st.tab);
        if (st.sched) cudaFree(st.sched);
        st.sched = nullptr;
        st.sched_bytes = 0;
        st.sched_valid = false;
        st.tab = nullptr;
        st.tab_bytes = 0;
        st.tab_L = -1;
        st.ws = st.dws = nullptr;
        st.maps_valid = false;
        st.ws_bytes = st.dws_bytes = 0;
    }
    cudaSetDevice(cur);
}

}  // extern "C"

// tp_mlp.cu -- the C ABI: handle, argument checks, workspace layout, plan choice.
//
// Every call checks its arguments on the host before launching anything:
// sizes and enums, 16-byte alignment, and that each device pointer lies inside
// one device allocation large enough for what the kernels will touch (so a
// wrong pointer is an error code, never an out-of-bounds access on the GPU).
#include <cuda.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <cmath>
#include <mutex>
#include <new>

#include "common.cuh"
#include "internal.h"

namespace tpmlp {

// Kernels whose dynamic shared-memory limit has been raised, per device.
namespace {
std::mutex g_attr_mutex;
struct AttrEntry {
    const void *fn;
    unsigned long long devices;   // bit d: done on device d (d < 64)
};
AttrEntry g_attr[64];
int g_attr_n = 0;
}  // namespace

bool smem_attr_done(const void *fn, int dev) {
    if (dev < 0 || dev >= 64) return false;
    std::lock_guard<std::mutex> lock(g_attr_mutex);
    for (int i = 0; i < g_attr_n; ++i)
        if (g_attr[i].fn == fn) return (g_attr[i].devices >> dev) & 1ull;
    return false;
}

void smem_attr_mark(const void *fn, int dev) {
    if (dev < 0 || dev >= 64) return;
    std::lock_guard<std::mutex> lock(g_attr_mutex);
    for (int i = 0; i < g_attr_n; ++i)
        if (g_attr[i].fn == fn) {
            g_attr[i].devices |= 1ull << dev;
            return;
        }
    if (g_attr_n < 64) g_attr[g_attr_n++] = AttrEntry{fn, 1ull << dev};   // full table: just re-set next time
}

}  // namespace tpmlp

using namespace tpmlp;

struct tp_mlp_s {
    int d_model, d_ff, d_out, tp, act, dtype, max_tokens;
    int num_sms;
    void *ws;
    size_t ws_bytes;
    int plan;            // forced tp_mlp_plan
    int splitk;          // tp_mlp_splitk: how the skinny tiling finishes split tiles
    int last_plan, last_launches;
    Marks marks;         // timing hook
    // split-K scratch each token count needs, precomputed at creation:
    // gemv_part[t] for t = 1..kGemvMaxTokens, tc_part[i] for skinny widths 16/32/64/128
    size_t gemv_part[kGemvMaxTokens + 1];
    size_t tc_part[4];
};

namespace tpmlp {

typedef CUresult (*PFN_getAddressRange)(CUdeviceptr *, size_t *, CUdeviceptr);

static PFN_getAddressRange address_range_fn() {
    static PFN_getAddressRange fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_getAddressRange>(p);
    });
    return fn;
}

int check_dev(const void *p, size_t bytes) {
    if (!p) return TP_MLP_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(p) & 15u) return TP_MLP_ERR_ALIGNMENT;
    PFN_getAddressRange fn = address_range_fn();
    if (!fn) return TP_MLP_ERR_CUDA;
    CUdeviceptr base = 0;
    size_t size = 0;
    if (fn(&base, &size, reinterpret_cast<CUdeviceptr>(p)) != CUDA_SUCCESS)
        return TP_MLP_ERR_INVALID_ARG;   // not memory of the current device's context
    if (reinterpret_cast<uintptr_t>(p) + bytes > base + size) return TP_MLP_ERR_SHAPE;
    return TP_MLP_OK;
}

typedef CUresult (*PFN_pointerGetAttribute)(void *, CUpointer_attribute, CUdeviceptr);

static PFN_pointerGetAttribute pointer_attribute_fn() {
    static PFN_pointerGetAttribute fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuPointerGetAttribute", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_pointerGetAttribute>(p);
    });
    return fn;
}

// A pointer a kernel of the current device may read or write `bytes` from:
// device memory of the current context (check_dev), or page-locked host
// memory mapped into the device's address space.  *dev is the address the
// kernel uses.
int check_reachable(const void *p, size_t bytes, const void **dev) {
    if (!p) return TP_MLP_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(p) & 15u) return TP_MLP_ERR_ALIGNMENT;
    PFN_pointerGetAttribute fn = pointer_attribute_fn();
    if (!fn) return TP_MLP_ERR_CUDA;
    const CUdeviceptr ptr = reinterpret_cast<CUdeviceptr>(p);
    unsigned type = 0;
    if (fn(&type, CU_POINTER_ATTRIBUTE_MEMORY_TYPE, ptr) != CUDA_SUCCESS)
        return TP_MLP_ERR_INVALID_ARG;   // memory CUDA does not know (pageable host memory)
    if (type != CU_MEMORYTYPE_HOST) {
        // device memory: of this device (another GPU's would need peer access)
        int ordinal = -1, cur = -1;
        if (fn(&ordinal, CU_POINTER_ATTRIBUTE_DEVICE_ORDINAL, ptr) == CUDA_SUCCESS && ordinal >= 0 &&
            (cudaGetDevice(&cur) != cudaSuccess || ordinal != cur))
            return TP_MLP_ERR_INVALID_ARG;
        *dev = p;
        return check_dev(p, bytes);
    }
    CUdeviceptr alias = 0, start = 0;
    size_t size = 0;
    if (fn(&alias, CU_POINTER_ATTRIBUTE_DEVICE_POINTER, ptr) != CUDA_SUCCESS ||
        fn(&start, CU_POINTER_ATTRIBUTE_RANGE_START_ADDR, ptr) != CUDA_SUCCESS ||
        fn(&size, CU_POINTER_ATTRIBUTE_RANGE_SIZE, ptr) != CUDA_SUCCESS)
        return TP_MLP_ERR_INVALID_ARG;   // not mapped for this device
    if (ptr < start || ptr + bytes > start + size) return TP_MLP_ERR_SHAPE;
    if (alias & 15u) return TP_MLP_ERR_ALIGNMENT;
    *dev = reinterpret_cast<const void *>(alias);
    return TP_MLP_OK;
}

}  // namespace tpmlp

namespace {

size_t elem_bytes(int dtype) { return dtype == TP_MLP_F32 ? 4 : 2; }

Problem problem_of(const tp_mlp_s *h, int tokens) {
    Problem p;
    p.T = tokens;
    p.d_in = h->d_model;
    p.d_ff = h->d_ff;
    p.d_out = h->d_out;
    p.tp = h->tp;
    p.fs = h->d_ff / h->tp;
    p.act = h->act;
    p.dtype = h->dtype;
    return p;
}

// Workspace layout:
//   [split-tile counters (GEMV and tcgen05 skinny share them) | status word]
//        (zeroed by set_workspace; the kernels leave the counters at zero)
//   [H: tokens x d_ff]
//   [split-tile partial sums]
size_t tile_counters_n(const tp_mlp_s *h) { return tile_counter_slots(problem_of(h, 1)); }
size_t counters_bytes(const tp_mlp_s *h) { return align256((tile_counters_n(h) + 1) * sizeof(unsigned)); }
int *status_word(const tp_mlp_s *h) {
    return reinterpret_cast<int *>(static_cast<unsigned *>(h->ws) + tile_counters_n(h));
}
size_t h_bytes(const tp_mlp_s *h, int tokens) {
    return align256((size_t)tokens * h->d_ff * elem_bytes(h->dtype));
}
// Largest split-K scratch any call with <= tokens tokens needs, so that a
// workspace sized for max_tokens serves every smaller call too.
size_t part_bytes(const tp_mlp_s *h, int tokens) {
    size_t m = 0;
    for (int t = 1; t <= tokens && t <= kGemvMaxTokens; ++t) m = h->gemv_part[t] > m ? h->gemv_part[t] : m;
    const int widths[4] = {16, 32, 64, 128};
    for (int i = 0; i < 4; ++i) {
        if (tokens >= 1 && (i == 0 || tokens > widths[i - 1]))
            m = h->tc_part[i] > m ? h->tc_part[i] : m;
    }
    return m;
}
size_t need_bytes(const tp_mlp_s *h, int tokens) {
    return counters_bytes(h) + h_bytes(h, tokens) + part_bytes(h, tokens);
}

int from_cuda(cudaError_t e) { return e == cudaSuccess ? TP_MLP_OK : TP_MLP_ERR_CUDA; }

// Checks shared by forward and partials (shard form).
int check_common(tp_mlp_t h, const void *x, int tokens, int tp_degree, int act) {
    if (!h) return TP_MLP_ERR_INVALID_ARG;
    if (tokens < 0 || tokens > h->max_tokens) return TP_MLP_ERR_SHAPE;
    if (tp_degree != h->tp) return TP_MLP_ERR_SHAPE;   // shards pair strictly, rank for rank
    if (act != h->act) return TP_MLP_ERR_INVALID_ARG;
    (void)x;
    return TP_MLP_OK;
}

int check_shards(tp_mlp_t h, const void *const *A, const void *const *B) {
    if (!A || !B) return TP_MLP_ERR_INVALID_ARG;
    const size_t e = elem_bytes(h->dtype);
    const size_t fs = (size_t)h->d_ff / h->tp;
    const size_t lda = h->act == TP_MLP_ACT_SWIGLU ? 2 * fs : fs;
    for (int i = 0; i < h->tp; ++i) {
        if (!A[i] || !B[i]) return TP_MLP_ERR_INVALID_ARG;
        if (((uintptr_t)A[i] | (uintptr_t)B[i]) & 15u) return TP_MLP_ERR_ALIGNMENT;
    }
    for (int i = 0; i < h->tp; ++i) {
        int s = check_dev(A[i], (size_t)h->d_model * lda * e);
        if (s) return s;
        s = check_dev(B[i], fs * h->d_out * e);
        if (s) return s;
    }
    return TP_MLP_OK;
}

int check_workspace(tp_mlp_t h, int tokens) {
    if (!h->ws || h->ws_bytes < need_bytes(h, tokens)) return TP_MLP_ERR_WORKSPACE;
    return TP_MLP_OK;
}

ShardPtrs to_ptrs(const void *const *arr, int n) {
    ShardPtrs s;
    memset(&s, 0, sizeof(s));
    for (int i = 0; i < n; ++i) s.p[i] = arr[i];
    return s;
}

}  // namespace

extern "C" {

int tp_mlp_create(tp_mlp_t *handle, int d_model, int d_ff, int d_out, int tp_degree, int act,
                  int dtype, int max_tokens) {
    if (!handle) return TP_MLP_ERR_INVALID_ARG;
    if (act != TP_MLP_ACT_TANH && act != TP_MLP_ACT_SWIGLU && act != TP_MLP_ACT_IDENTITY)
        return TP_MLP_ERR_INVALID_ARG;
    if (dtype != TP_MLP_F32 && dtype != TP_MLP_BF16) return TP_MLP_ERR_INVALID_ARG;
    if (d_model < 1 || d_ff < 1 || d_out < 1 || max_tokens < 1) return TP_MLP_ERR_SHAPE;
    if (tp_degree < 1 || tp_degree > kMaxTp || d_ff % tp_degree != 0) return TP_MLP_ERR_SHAPE;
    // keep every index inside 32-bit ints where the kernels use them
    if ((long long)max_tokens * d_ff > (1LL << 31) || (long long)max_tokens * d_model > (1LL << 31) ||
        (long long)max_tokens * d_out > (1LL << 31))
        return TP_MLP_ERR_SHAPE;
    tp_mlp_s *h = new (std::nothrow) tp_mlp_s;
    if (!h) return TP_MLP_ERR_INVALID_ARG;
    h->d_model = d_model;
    h->d_ff = d_ff;
    h->d_out = d_out;
    h->tp = tp_degree;
    h->act = act;
    h->dtype = dtype;
    h->max_tokens = max_tokens;
    h->ws = nullptr;
    h->ws_bytes = 0;
    h->plan = TP_MLP_PLAN_AUTO;
    h->splitk = TP_MLP_SPLITK_AUTO;
    h->last_plan = -1;
    h->last_launches = -1;
    memset(&h->marks, 0, sizeof(h->marks));
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && sms > 0)
        h->num_sms = sms;
    else {
        cudaGetLastError();
        h->num_sms = 148;   // B200; only sizes split-K scratch
    }
    h->gemv_part[0] = 0;
    for (int t = 1; t <= kGemvMaxTokens; ++t)
        h->gemv_part[t] = t <= max_tokens ? gemv_workspace_bytes(problem_of(h, t), h->num_sms) : 0;
    const int widths[4] = {16, 32, 64, 128};
    for (int i = 0; i < 4; ++i) {
        const int t = widths[i] < max_tokens ? widths[i] : max_tokens;
        if (i > 0 && max_tokens <= widths[i - 1]) {
            h->tc_part[i] = 0;
            continue;
        }
        Problem p = problem_of(h, t);
        size_t m = tc_workspace_bytes(p, h->num_sms);
        // the cross-GPU step runs one rank's shards alone (tp 1, d_ff / tp features)
        Problem p1 = p;
        p1.tp = 1;
        p1.d_ff = p.fs;
        if (p.fs % 64 == 0) {
            const size_t m1 = tc_workspace_bytes(p1, h->num_sms);
            m = m1 > m ? m1 : m;
        }
        h->tc_part[i] = m;
    }
    *handle = h;
    return TP_MLP_OK;
}

int tp_mlp_destroy(tp_mlp_t h) {
    delete h;
    return TP_MLP_OK;
}

size_t tp_mlp_workspace_bytes(tp_mlp_t h, int tokens) {
    if (!h || tokens < 0 || tokens > h->max_tokens) return 0;
    return need_bytes(h, tokens);
}

int tp_mlp_set_workspace(tp_mlp_t h, void *dev_ptr, size_t bytes) {
    if (!h) return TP_MLP_ERR_INVALID_ARG;
    if (!dev_ptr) {
        h->ws = nullptr;
        h->ws_bytes = 0;
        return TP_MLP_OK;
    }
    if (bytes < need_bytes(h, 0)) return TP_MLP_ERR_WORKSPACE;
    int s = check_dev(dev_ptr, bytes);
    if (s) return s;
    // the memset runs on the legacy stream: wait for it, so that a forward on
    // any stream sees zeroed counters
    if (cudaMemset(dev_ptr, 0, counters_bytes(h)) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess)
        return TP_MLP_ERR_CUDA;
    h->ws = dev_ptr;
    h->ws_bytes = bytes;
    return TP_MLP_OK;
}

static int run_shard_form(tp_mlp_t h, const void *x, int tokens, const void *const *A,
                          const void *const *B, int tp_degree, int act, void *out, float *partials,
                          tp_mlp_stream_t stream) {
    int s = check_common(h, x, tokens, tp_degree, act);
    if (s) return s;
    Problem p = problem_of(h, tokens);
    // The forward and the partials read the shards straight into the tcgen05
    // kernels when the shape allows (bf16, f_s % 64 == 0); other shapes use the
    // CUDA-core kernels.  The GEMV needs the packed layout.
    const bool tc_ok = tc_raw_supported(p);
    int plan = h->plan;
    if (plan == TP_MLP_PLAN_AUTO) plan = tc_ok ? TP_MLP_PLAN_TC : TP_MLP_PLAN_SIMT;
    // Up to 128 tokens: the two-kernel skinny tiling.  The fused kernel also
    // takes the shard form (TP_MLP_PLAN_TC_FUSED) but measured slower on it:
    // its 256-row first-projection tiles are split, and inside the fused
    // kernel their slots must be added at the end of the first projection,
    // where the reduction kernel spreads that work over the GPU (sweep d 4096 /
    // f 16384, tp 8, 16 / 64 / 128 tokens: 53.5 / 66.8 / 81.8 against 52.6 /
    // 57.6 / 67.2 us; decode bs32 231 against 225).
    if (plan == TP_MLP_PLAN_TC)
        plan = tokens <= kTcSkinnyMaxTokens ? TP_MLP_PLAN_TC_SKINNY
               : tokens < kTcWide256MinTokens ? TP_MLP_PLAN_TC_WIDE
                                              : TP_MLP_PLAN_TC_WIDE256;
    const bool is_tc = plan == TP_MLP_PLAN_TC_WIDE || plan == TP_MLP_PLAN_TC_SKINNY || plan == TP_MLP_PLAN_TC_WIDE256 ||
                       (plan == TP_MLP_PLAN_TC_FUSED && !partials);
    if (plan != TP_MLP_PLAN_SIMT && !is_tc) return TP_MLP_ERR_UNSUPPORTED;   // (the pair tiling needs packed weights)
    if (is_tc && tokens > 0 &&
        (!tc_ok || (plan == TP_MLP_PLAN_TC_SKINNY && tokens > kTcSkinnyMaxTokens) ||
         (plan == TP_MLP_PLAN_TC_FUSED && !fused_supported(p, true))))
        return TP_MLP_ERR_UNSUPPORTED;
    if (tokens == 0) {
        h->last_plan = plan;
        h->last_launches = 0;
        return TP_MLP_OK;
    }
    const size_t e = elem_bytes(h->dtype);
    if ((s = check_dev(x, (size_t)tokens * h->d_model * e))) return s;
    if (partials) {
        if ((s = check_dev(partials, (size_t)h->tp * tokens * h->d_out * sizeof(float)))) return s;
    } else if ((s = check_dev(out, (size_t)tokens * h->d_out * e))) {
        return s;
    }
    if ((s = check_shards(h, A, B))) return s;
    if ((s = check_workspace(h, tokens))) return s;
    char *ws = static_cast<char *>(h->ws);
    void *hbuf = ws + counters_bytes(h);
    const ShardPtrs a = to_ptrs(A, h->tp), b = to_ptrs(B, h->tp);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t ce;
    int launches = 2;
    if (is_tc) {
        const int tiling = plan == TP_MLP_PLAN_TC_SKINNY  ? kTilingSkinny
                           : plan == TP_MLP_PLAN_TC_FUSED ? kTilingFused
                           : plan == TP_MLP_PLAN_TC_WIDE  ? kTilingWide128
                                                          : kTilingWide256;
        float *part = reinterpret_cast<float *>(ws + counters_bytes(h) + h_bytes(h, tokens));
        ce = launch_tc(p, tiling, x, nullptr, nullptr, &a, &b, hbuf, out, part, reinterpret_cast<unsigned *>(ws),
                       status_word(h), h->num_sms, st, h->marks, h->splitk, &launches, partials);
    } else {
        ce = launch_simt(p, false, x, a, b, hbuf, out, partials, st, h->marks);
    }
    if (ce != cudaSuccess) return TP_MLP_ERR_CUDA;
    h->last_plan = plan;
    h->last_launches = launches;
    return TP_MLP_OK;
}

int tp_mlp_forward(tp_mlp_t h, const void *x, int tokens, const void *const *A_shards,
                   const void *const *B_shards, int tp_degree, int act, void *out,
                   tp_mlp_stream_t stream) {
    return run_shard_form(h, x, tokens, A_shards, B_shards, tp_degree, act, out, nullptr, stream);
}

int tp_mlp_partials(tp_mlp_t h, const void *x, int tokens, const void *const *A_shards,
                    const void *const *B_shards, int tp_degree, int act, float *partials,
                    tp_mlp_stream_t stream) {
    if (!partials && h && tokens > 0) return TP_MLP_ERR_INVALID_ARG;
    return run_shard_form(h, x, tokens, A_shards, B_shards, tp_degree, act, nullptr, partials, stream);
}

size_t tp_mlp_packed_bytes(tp_mlp_t h) {
    if (!h) return 0;
    return packed_total_bytes(problem_of(h, 0));
}

static int pack_common(tp_mlp_t h, const void *const *A, const void *const *B, const void *packed,
                       bool unpack, tp_mlp_stream_t stream) {
    if (!h) return TP_MLP_ERR_INVALID_ARG;
    int s = check_shards(h, A, B);
    if (s) return s;
    if ((s = check_dev(packed, tp_mlp_packed_bytes(h)))) return s;
    Problem p = problem_of(h, 0);
    return from_cuda(launch_pack(p, to_ptrs(A, h->tp), to_ptrs(B, h->tp), const_cast<void *>(packed),
                                 unpack, reinterpret_cast<cudaStream_t>(stream)));
}

int tp_mlp_pack(tp_mlp_t h, const void *const *A_shards, const void *const *B_shards, void *packed,
                tp_mlp_stream_t stream) {
    return pack_common(h, A_shards, B_shards, packed, false, stream);
}

int tp_mlp_unpack(tp_mlp_t h, const void *packed, void *const *A_shards, void *const *B_shards,
                  tp_mlp_stream_t stream) {
    return pack_common(h, A_shards, B_shards, packed, true, stream);
}

int tp_mlp_forward_packed(tp_mlp_t h, const void *x, int tokens, const void *packed, void *out,
                          tp_mlp_stream_t stream) {
    if (!h) return TP_MLP_ERR_INVALID_ARG;
    if (tokens < 0 || tokens > h->max_tokens) return TP_MLP_ERR_SHAPE;
    Problem p = problem_of(h, tokens);
    // plan choice (measured on B200 at d_model 8192, d_ff 28672): the CUDA-core
    // GEMV for 1 token; from 2 tokens on the tensor-core skinny tiling streams
    // the weights as fast and its arithmetic stays hidden -- both projections
    // in one persistent launch, which measured 1-4 % faster than two kernels
    // at 2-128 tokens (decode and the d 4096 / f 16384 sweep); wide beyond
    // 128, pairs of CTAs from 512 to 4096 tokens, two-tile pairs above.
    int plan = h->plan;
    const bool tc_ok = tc_supported(p);
    auto tc_tiling = [&](int t) {
        return t <= kTcSkinnyMaxTokens ? (fused_supported(p, false) ? TP_MLP_PLAN_TC_FUSED : TP_MLP_PLAN_TC_SKINNY)
               : t < kTcPairMinTokens  ? TP_MLP_PLAN_TC_WIDE
               : t <= kTcPairMaxTokens ? TP_MLP_PLAN_TC_PAIR
                                       : TP_MLP_PLAN_TC_PAIR2;
    };
    if (plan == TP_MLP_PLAN_AUTO) {
        if (gemv_supported(p) && (tokens <= 1 || !tc_ok)) plan = TP_MLP_PLAN_GEMV;
        else if (tc_ok) plan = tc_tiling(tokens);
        else plan = TP_MLP_PLAN_SIMT;
    } else if (plan == TP_MLP_PLAN_TC) {
        plan = tc_tiling(tokens);
    }
    const bool is_tc = plan == TP_MLP_PLAN_TC_WIDE || plan == TP_MLP_PLAN_TC_SKINNY ||
                       plan == TP_MLP_PLAN_TC_WIDE256 || plan == TP_MLP_PLAN_TC_PAIR || plan == TP_MLP_PLAN_TC_PAIR2 ||
                       plan == TP_MLP_PLAN_TC_FUSED;
    if (tokens > 0) {
        if (plan == TP_MLP_PLAN_GEMV && !gemv_supported(p)) return TP_MLP_ERR_UNSUPPORTED;
        if (plan == TP_MLP_PLAN_TC_FUSED && !fused_supported(p, false)) return TP_MLP_ERR_UNSUPPORTED;
        if (is_tc && !tc_ok) return TP_MLP_ERR_UNSUPPORTED;
        if (plan == TP_MLP_PLAN_TC_SKINNY && tokens > kTcSkinnyMaxTokens) return TP_MLP_ERR_UNSUPPORTED;
    }
    if (tokens == 0) {
        h->last_plan = plan;
        h->last_launches = 0;
        return TP_MLP_OK;
    }
    const size_t e = elem_bytes(h->dtype);
    int s;
    if ((s = check_dev(x, (size_t)tokens * h->d_model * e))) return s;
    if ((s = check_dev(out, (size_t)tokens * h->d_out * e))) return s;
    if ((s = check_dev(packed, tp_mlp_packed_bytes(h)))) return s;
    if ((s = check_workspace(h, tokens))) return s;
    char *ws = static_cast<char *>(h->ws);
    unsigned *counters = reinterpret_cast<unsigned *>(ws);
    void *hbuf = ws + counters_bytes(h);
    float *part = reinterpret_cast<float *>(ws + counters_bytes(h) + h_bytes(h, tokens));
    const void *w1p = packed;
    const void *w2p = static_cast<const char *>(packed) + packed_part2_offset(p);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t ce;
    int launches = 2;
    if (plan == TP_MLP_PLAN_GEMV) {
        ce = launch_gemv(p, x, w1p, w2p, hbuf, out, part, counters, status_word(h), h->num_sms, st, h->marks,
                         &launches);
    } else if (is_tc) {
        const int tiling = plan == TP_MLP_PLAN_TC_SKINNY ? kTilingSkinny
                           : plan == TP_MLP_PLAN_TC_WIDE ? kTilingWide128
                           : plan == TP_MLP_PLAN_TC_PAIR ? kTilingPair
                           : plan == TP_MLP_PLAN_TC_PAIR2 ? kTilingPair2
                           : plan == TP_MLP_PLAN_TC_FUSED ? kTilingFused : kTilingWide256;
        ce = launch_tc(p, tiling, x, w1p, w2p, nullptr, nullptr, hbuf, out, part, counters, status_word(h),
                       h->num_sms, st, h->marks, h->splitk, &launches);
    } else {
        ShardPtrs a, b;
        memset(&a, 0, sizeof(a));
        memset(&b, 0, sizeof(b));
        a.p[0] = w1p;
        b.p[0] = w2p;
        ce = launch_simt(p, true, x, a, b, hbuf, out, nullptr, st, h->marks);
    }
    if (ce != cudaSuccess) return TP_MLP_ERR_CUDA;
    h->last_plan = plan;
    h->last_launches = launches;
    return TP_MLP_OK;
}

int tp_mlp_get_device_status(tp_mlp_t h) {
    if (!h) return TP_MLP_ERR_INVALID_ARG;
    if (!h->ws) return TP_MLP_ERR_WORKSPACE;
    int v = 0;
    if (cudaMemcpy(&v, status_word(h), sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return TP_MLP_ERR_CUDA;
    if (v == 0) return TP_MLP_OK;
    // A kernel gave up a bounded wait: its CTAs left early, so split-tile
    // counters may be left part-way.  Zero them with the status word, so the
    // next call starts from the state set_workspace leaves.
    if (cudaMemset(h->ws, 0, counters_bytes(h)) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess)
        return TP_MLP_ERR_CUDA;
    return TP_MLP_ERR_TIMEOUT;
}

int tp_mlp_selftest_bounded_wait(tp_mlp_t h, unsigned wait_us, tp_mlp_stream_t stream) {
    if (!h) return TP_MLP_ERR_INVALID_ARG;
    if (!h->ws) return TP_MLP_ERR_WORKSPACE;
    if (wait_us == 0 || wait_us > 100000) return TP_MLP_ERR_INVALID_ARG;
    return from_cuda(launch_bounded_wait_selftest(status_word(h), wait_us,
                                                  reinterpret_cast<cudaStream_t>(stream)));
}

int tp_mlp_set_plan(tp_mlp_t h, int plan) {
    if (!h) return TP_MLP_ERR_INVALID_ARG;
    if (plan < TP_MLP_PLAN_AUTO || plan > TP_MLP_PLAN_TC_FUSED) return TP_MLP_ERR_INVALID_ARG;
    h->plan = plan;
    return TP_MLP_OK;
}

int tp_mlp_allreduce_residual_rmsnorm(const float *partials, int tp_degree, int tokens, int d,
                                      const void *residual, const void *gamma, float eps, int dtype,
                                      void *y, void *residual_out, tp_mlp_stream_t stream) {
    if (tp_degree < 1 || tp_degree > kMaxTp || tokens < 0) return TP_MLP_ERR_SHAPE;
    if (d < 4 || d > kNormMaxWidth || d % 4 != 0) return TP_MLP_ERR_SHAPE;
    if (!(eps >= 0.f) || !std::isfinite(eps)) return TP_MLP_ERR_INVALID_ARG;
    if (dtype != TP_MLP_F32 && dtype != TP_MLP_BF16) return TP_MLP_ERR_INVALID_ARG;
    if (tokens == 0) return TP_MLP_OK;   // empty tensors may carry null pointers
    if (!partials || !residual || !gamma || !y || !residual_out) return TP_MLP_ERR_INVALID_ARG;
    const size_t e = elem_bytes(dtype), n = (size_t)tokens * d;
    int s;
    if ((s = check_dev(partials, (size_t)tp_degree * n * sizeof(float)))) return s;
    if ((s = check_dev(residual, n * e))) return s;
    if ((s = check_dev(gamma, (size_t)d * e))) return s;
    if ((s = check_dev(y, n * e))) return s;
    if ((s = check_dev(residual_out, n * e))) return s;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
        return TP_MLP_ERR_CUDA;
    return from_cuda(launch_allreduce_norm(partials, tp_degree, tokens, d, residual, gamma, eps, dtype, y,
                                           residual_out, sms, reinterpret_cast<cudaStream_t>(stream)));
}

int tp_mlp_merge_attention_partials(int tp_degree, int rows, int head_dim, const float *maximum,
                                    const float *exp_sum, const void *weighted, int dtype, void *out,
                                    tp_mlp_stream_t stream) {
    if (tp_degree < 1 || tp_degree > kMaxTp || rows < 0) return TP_MLP_ERR_SHAPE;
    if (head_dim < 4 || head_dim > kMergeMaxHeadDim || head_dim % 4 != 0) return TP_MLP_ERR_SHAPE;
    if (dtype != TP_MLP_F32 && dtype != TP_MLP_BF16) return TP_MLP_ERR_INVALID_ARG;
    if (rows == 0) return TP_MLP_OK;   // empty tensors may carry null pointers
    if (!maximum || !exp_sum || !weighted || !out) return TP_MLP_ERR_INVALID_ARG;
    const size_t e = elem_bytes(dtype), pr = (size_t)tp_degree * rows;
    int s;
    if ((s = check_dev(maximum, pr * sizeof(float)))) return s;
    if ((s = check_dev(exp_sum, pr * sizeof(float)))) return s;
    if ((s = check_dev(weighted, pr * head_dim * e))) return s;
    if ((s = check_dev(out, (size_t)rows * head_dim * e))) return s;
    return from_cuda(launch_attn_merge(tp_degree, rows, head_dim, maximum, exp_sum, weighted, dtype, out,
                                       reinterpret_cast<cudaStream_t>(stream)));
}

int tp_mlp_copy_async(void *dst, const void *src, size_t bytes, tp_mlp_stream_t stream) {
    if (bytes == 0) return TP_MLP_OK;
    if (!dst || !src) return TP_MLP_ERR_INVALID_ARG;
    const uintptr_t a = reinterpret_cast<uintptr_t>(src), b = reinterpret_cast<uintptr_t>(dst);
    if ((a | b) & 15u) return TP_MLP_ERR_ALIGNMENT;
    const void *s_dev = nullptr, *d_dev = nullptr;
    int s;
    if ((s = check_reachable(src, bytes, &s_dev))) return s;
    if ((s = check_reachable(dst, bytes, &d_dev))) return s;
    if (a < b + bytes && b < a + bytes) return TP_MLP_ERR_INVALID_ARG;   // overlapping ranges
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (bytes > kCopyKernelMaxBytes) return from_cuda(cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDefault, st));
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
        return TP_MLP_ERR_CUDA;
    return from_cuda(launch_copy(const_cast<void *>(d_dev), s_dev, bytes, sms, st));
}

// Exchange buffer: [control + flags | receive rows | gathered rows (sequence parallelism)].
static size_t xgpu_recv_bytes(const tp_mlp_s *h) { return align256(2 * (size_t)h->tp * h->max_tokens * h->d_out * 2); }

size_t tp_mlp_xgpu_comm_bytes(tp_mlp_t h) {
    if (!h) return 0;
    const Problem p = problem_of(h, 0);
    return xgpu_header_bytes(p) + xgpu_recv_bytes(h) + align256((size_t)h->max_tokens * h->d_model * 2);
}

static int xgpu_common(tp_mlp_t h, bool sp, int rank0, int nranks, const void *const *x, int tokens,
                       const void *const *A_local, const void *const *B_local, void *const *comm,
                       void *const *outs, tp_mlp_stream_t stream) {
    if (!h) return TP_MLP_ERR_INVALID_ARG;
    Problem p = problem_of(h, tokens);
    if (h->dtype != TP_MLP_BF16 || !tc_raw_supported(p) || h->d_model % 8) return TP_MLP_ERR_UNSUPPORTED;
    if (tokens < 0 || tokens > h->max_tokens || tokens > kTcSkinnyMaxTokens) return TP_MLP_ERR_SHAPE;
    if (sp && tokens % h->tp) return TP_MLP_ERR_SHAPE;
    if (nranks < 1 || rank0 < 0 || rank0 + nranks > h->tp) return TP_MLP_ERR_SHAPE;
    if (tokens == 0) return TP_MLP_OK;   // launches nothing (empty tensors may carry null pointers)
    if (!x || !A_local || !B_local || !comm || !outs) return TP_MLP_ERR_INVALID_ARG;
    const size_t fs = (size_t)h->d_ff / h->tp;
    const size_t lda = h->act == TP_MLP_ACT_SWIGLU ? 2 * fs : fs;
    const size_t rows_in = sp ? tokens / h->tp : tokens, rows_out = rows_in;
    int s;
    for (int i = 0; i < (sp ? nranks : 1); ++i)
        if ((s = check_dev(x[i], rows_in * h->d_model * 2))) return s;
    for (int i = 0; i < nranks; ++i) {
        if ((s = check_dev(A_local[i], (size_t)h->d_model * lda * 2))) return s;
        if ((s = check_dev(B_local[i], fs * h->d_out * 2))) return s;
        if ((s = check_dev(outs[i], rows_out * h->d_out * 2))) return s;
    }
    const size_t cb = tp_mlp_xgpu_comm_bytes(h);
    for (int r = 0; r < h->tp; ++r) {
        if (!comm[r]) return TP_MLP_ERR_INVALID_ARG;
        if (reinterpret_cast<uintptr_t>(comm[r]) & 15u) return TP_MLP_ERR_ALIGNMENT;
        // local buffers are checked in full; a peer's may be a mapping of another GPU's memory
        if (r >= rank0 && r < rank0 + nranks && (s = check_dev(comm[r], cb))) return s;
    }
    Problem pl = p;
    pl.tp = nranks;
    pl.d_ff = nranks * p.fs;
    const size_t hb = align256((size_t)tokens * pl.d_ff * 2);
    const size_t need = counters_bytes(h) + hb + tc_workspace_bytes(pl, h->num_sms);
    if (!h->ws || h->ws_bytes < need) return TP_MLP_ERR_WORKSPACE;
    char *ws = static_cast<char *>(h->ws);
    XgpuArgs xa;
    memset(&xa, 0, sizeof(xa));
    for (int r = 0; r < h->tp; ++r) xa.comm[r] = comm[r];
    for (int i = 0; i < nranks; ++i) xa.outs[i] = outs[i];
    xa.recv_off = xgpu_header_bytes(p);
    xa.rows = h->max_tokens;
    const ShardPtrs a = to_ptrs(A_local, nranks), b = to_ptrs(B_local, nranks);
    void *hbuf = ws + counters_bytes(h);
    float *part = reinterpret_cast<float *>(ws + counters_bytes(h) + hb);
    unsigned *cnt = reinterpret_cast<unsigned *>(ws);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int launches = 0;
    const cudaError_t ce =
        sp ? launch_xgpu_sp(p, rank0, nranks, x, a, b, hbuf, part, cnt, status_word(h), h->num_sms, st, xa,
                            xa.recv_off + xgpu_recv_bytes(h), &launches)
           : launch_xgpu(p, rank0, nranks, x[0], a, b, hbuf, part, cnt, status_word(h), h->num_sms, st, xa,
                         &launches);
    if (ce == cudaErrorNotSupported) {
        cudaGetLastError();
        return TP_MLP_ERR_UNSUPPORTED;
    }
    if (ce != cudaSuccess) return TP_MLP_ERR_CUDA;
    h->last_plan = TP_MLP_PLAN_TC_SKINNY;
    h->last_launches = launches;
    return TP_MLP_OK;
}

int tp_mlp_xgpu_forward(tp_mlp_t h, int rank0, int nranks, const void *x, int tokens,
                        const void *const *A_local, const void *const *B_local, void *const *comm,
                        void *const *outs, tp_mlp_stream_t stream) {
    const void *xs[1] = {x};
    return xgpu_common(h, false, rank0, nranks, xs, tokens, A_local, B_local, comm, outs, stream);
}

int tp_mlp_xgpu_sp_forward(tp_mlp_t h, int rank0, int nranks, const void *const *x_local, int tokens,
                           const void *const *A_local, const void *const *B_local, void *const *comm,
                           void *const *outs, tp_mlp_stream_t stream) {
    return xgpu_common(h, true, rank0, nranks, x_local, tokens, A_local, B_local, comm, outs, stream);
}

int tp_mlp_ipc_get_handle(const void *dev_ptr, void *handle, size_t *offset) {
    if (!dev_ptr || !handle || !offset) return TP_MLP_ERR_INVALID_ARG;
    PFN_getAddressRange fn = address_range_fn();
    if (!fn) return TP_MLP_ERR_CUDA;
    CUdeviceptr base = 0;
    size_t size = 0;
    if (fn(&base, &size, reinterpret_cast<CUdeviceptr>(dev_ptr)) != CUDA_SUCCESS) return TP_MLP_ERR_INVALID_ARG;
    cudaIpcMemHandle_t hd;
    if (cudaIpcGetMemHandle(&hd, reinterpret_cast<void *>(base)) != cudaSuccess) {
        cudaGetLastError();
        return TP_MLP_ERR_CUDA;
    }
    memcpy(handle, &hd, sizeof(hd));
    *offset = reinterpret_cast<uintptr_t>(dev_ptr) - (uintptr_t)base;
    return TP_MLP_OK;
}

int tp_mlp_ipc_open_handle(const void *handle, size_t offset, void **dev_ptr) {
    if (!handle || !dev_ptr) return TP_MLP_ERR_INVALID_ARG;
    cudaIpcMemHandle_t hd;
    memcpy(&hd, handle, sizeof(hd));
    void *base = nullptr;
    if (cudaIpcOpenMemHandle(&base, hd, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
        cudaGetLastError();
        return TP_MLP_ERR_CUDA;
    }
    *dev_ptr = static_cast<char *>(base) + offset;
    return TP_MLP_OK;
}

int tp_mlp_ipc_close_handle(void *dev_ptr, size_t offset) {
    if (!dev_ptr) return TP_MLP_ERR_INVALID_ARG;
    if (cudaIpcCloseMemHandle(static_cast<char *>(dev_ptr) - offset) != cudaSuccess) {
        cudaGetLastError();
        return TP_MLP_ERR_CUDA;
    }
    return TP_MLP_OK;
}

int tp_mlp_set_splitk(tp_mlp_t h, int mode) {
    if (!h) return TP_MLP_ERR_INVALID_ARG;
    if (mode < TP_MLP_SPLITK_AUTO || mode > TP_MLP_SPLITK_CLUSTER) return TP_MLP_ERR_INVALID_ARG;
    h->splitk = mode;
    return TP_MLP_OK;
}

int tp_mlp_set_profile_events(tp_mlp_t h, void *const *events, int n) {
    if (!h || n < 0 || n > 8) return TP_MLP_ERR_INVALID_ARG;
    memset(&h->marks, 0, sizeof(h->marks));
    if (!events || n == 0) return TP_MLP_OK;
    for (int i = 0; i < n; ++i) h->marks.ev[i] = static_cast<cudaEvent_t>(events[i]);
    h->marks.n = n;
    return TP_MLP_OK;
}

int tp_mlp_last_plan(tp_mlp_t h) { return h ? h->last_plan : -1; }
int tp_mlp_last_launches(tp_mlp_t h) { return h ? h->last_launches : -1; }

const char *tp_mlp_status_string(int status) {
    switch (status) {
        case TP_MLP_OK: return "ok";
        case TP_MLP_ERR_INVALID_ARG: return "invalid argument";
        case TP_MLP_ERR_SHAPE: return "shape mismatch";
        case TP_MLP_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
        case TP_MLP_ERR_UNSUPPORTED: return "unsupported by the library";
        case TP_MLP_ERR_CUDA: return "CUDA error";
        case TP_MLP_ERR_TIMEOUT: return "device wait timed out";
        case TP_MLP_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

}  // extern "C"

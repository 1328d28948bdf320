// profile.cu -- launch counting and opt-in per-launch event timing
// (wide_profile_* in wide.h).
#include <atomic>
#include <cuda_runtime.h>
#include <mutex>
#include <vector>

#include "host.h"
#include "wide.h"

namespace wide {
namespace {

std::atomic<int64_t> g_launches{0};
std::atomic<bool> g_on{false};
std::mutex g_mu;

struct Record {
    int32_t kid;
    cudaEvent_t begin, end;
};
std::vector<Record> g_pool;   // events created once
int g_used = 0;

}  // namespace

LaunchScope::LaunchScope(int32_t kernel_id, cudaStream_t s) : slot_(-1), s_(s)
{
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (!g_on.load(std::memory_order_relaxed))
        return;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_used >= (int)g_pool.size())
        return;
    slot_ = g_used++;
    g_pool[slot_].kid = kernel_id;
    cudaEventRecord(g_pool[slot_].begin, s_);
}

LaunchScope::~LaunchScope()
{
    if (slot_ >= 0)
        cudaEventRecord(g_pool[slot_].end, s_);
}

}  // namespace wide

using namespace wide;

extern "C" {

int wide_profile_start(int32_t max_records)
{
    if (max_records <= 0 || max_records > 65536)
        return WIDE_EINVAL;
    std::lock_guard<std::mutex> lock(g_mu);
    while ((int)g_pool.size() < max_records) {
        Record r{0, nullptr, nullptr};
        if (cudaEventCreate(&r.begin) != cudaSuccess || cudaEventCreate(&r.end) != cudaSuccess)
            return WIDE_CUDA_FAIL();
        g_pool.push_back(r);
    }
    g_used = 0;
    g_on.store(true);
    return WIDE_OK;
}

int wide_profile_stop(void)
{
    g_on.store(false);
    return WIDE_OK;
}

int wide_profile_read(int32_t *kernel_ids, float *ms, int32_t max, int32_t *n)
{
    if (!kernel_ids || !ms || !n || max < 0)
        return WIDE_EINVAL;
    std::lock_guard<std::mutex> lock(g_mu);
    int k = 0;
    for (int i = 0; i < g_used && k < max; ++i) {
        if (cudaEventSynchronize(g_pool[i].end) != cudaSuccess)
            return WIDE_CUDA_FAIL();
        float t = 0.f;
        if (cudaEventElapsedTime(&t, g_pool[i].begin, g_pool[i].end) != cudaSuccess)
            return WIDE_CUDA_FAIL();
        kernel_ids[k] = g_pool[i].kid;
        ms[k] = t;
        ++k;
    }
    *n = k;
    g_used = 0;
    return WIDE_OK;
}

const char *wide_kernel_name(int32_t id)
{
    switch (id) {
    case KID_REORDER_PARTITION_RANK:
        return "reorder_partition_rank";
    case KID_REORDER_FINISH:
        return "reorder_finish";
    case KID_DECODE_GATEUP:
        return "decode_gateup_gemv";
    case KID_DECODE_DOWN:
        return "decode_down_gemv";
    case KID_PREFILL_GATEUP:
        return "prefill_gateup_tcgen05";
    case KID_PREFILL_DOWN:
        return "prefill_down_tcgen05";
    case KID_DECODE_QKV:
        return "decode_qkv_rope_gemv";
    case KID_DECODE_ATTN:
        return "decode_attention";
    case KID_RMSNORM:
        return "rmsnorm";
    case KID_PREFILL_Q:
        return "prefill_q_rope_tcgen05";
    case KID_PREFILL_KV:
        return "prefill_kv_rope_tcgen05";
    case KID_PREFILL_ATTN:
        return "prefill_attention_tcgen05";
    case KID_PREFILL_OPROJ:
        return "prefill_oproj_tcgen05";
    case KID_ROUTER:
        return "router_tcgen05";
    case KID_ROUTER_SMALL:
        return "router_small_gemv";
    case KID_DECODE_FFN_SPLIT:
        return "decode_ffn_split_gemv";
    case KID_DECODE_FFN_TC:
        return "decode_ffn_tcgen05";
    case KID_FFN_PACK:
        return "ffn_pack";
    default:
        return "?";
    }
}

int64_t wide_launch_count(void) { return g_launches.load(); }

}  // extern "C"

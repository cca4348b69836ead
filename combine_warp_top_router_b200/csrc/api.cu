// api.cu -- status strings, version and launch accounting of libmoedispatch.
#include <atomic>

#include "common.cuh"

namespace md {
static std::atomic<uint64_t> g_launches{0};
static std::atomic<uint64_t> g_memsets{0};
void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }
void count_memsets(int n) { g_memsets.fetch_add((uint64_t)n, std::memory_order_relaxed); }

// Fault injection for tests (md_set_test_hooks): a short poll limit and one
// publish / one copy left out, so that a bounded wait runs out.
static std::atomic<long long> g_poll_limit{0};
static std::atomic<int> g_layout_skip_tile{-1};
static std::atomic<long long> g_expand_skip_unit{-1};
long long hook_poll_limit(long long dflt)
{
    const long long v = g_poll_limit.load(std::memory_order_relaxed);
    return v > 0 ? v : dflt;
}
int hook_layout_skip_tile() { return g_layout_skip_tile.load(std::memory_order_relaxed); }
long long hook_expand_skip_unit() { return g_expand_skip_unit.load(std::memory_order_relaxed); }

static std::atomic<int> g_permute_path{MD_PERMUTE_AUTO};
int permute_path() { return g_permute_path.load(std::memory_order_relaxed); }
static std::atomic<int> g_layout_path{MD_LAYOUT_AUTO};
int layout_path() { return g_layout_path.load(std::memory_order_relaxed); }
}  // namespace md

extern "C" int md_set_layout_path(int path)
{
    if (path != MD_LAYOUT_AUTO && path != MD_LAYOUT_COOPERATIVE && path != MD_LAYOUT_SPLIT)
        return MD_ERR_ARG;
    md::g_layout_path.store(path, std::memory_order_relaxed);
    return MD_OK;
}

extern "C" int md_set_permute_path(int path)
{
    if (path != MD_PERMUTE_AUTO && path != MD_PERMUTE_BULK && path != MD_PERMUTE_VECTOR)
        return MD_ERR_ARG;
    md::g_permute_path.store(path, std::memory_order_relaxed);
    return MD_OK;
}

extern "C" void md_set_test_hooks(long long poll_limit, int layout_skip_tile,
                                  long long expand_skip_unit)
{
    md::g_poll_limit.store(poll_limit, std::memory_order_relaxed);
    md::g_layout_skip_tile.store(layout_skip_tile, std::memory_order_relaxed);
    md::g_expand_skip_unit.store(expand_skip_unit, std::memory_order_relaxed);
}

extern "C" const char *md_status_string(int status)
{
    switch (status) {
    case MD_OK: return "MD_OK";
    case MD_ERR_ARG: return "MD_ERR_ARG: invalid argument";
    case MD_ERR_UNSUPPORTED: return "MD_ERR_UNSUPPORTED: size outside the supported limits";
    case MD_ERR_CUDA: return "MD_ERR_CUDA: a CUDA launch or memset failed";
    case MD_ERR_WORKSPACE: return "MD_ERR_WORKSPACE: workspace too small";
    case MD_ERR_DATA: return "MD_ERR_DATA: invalid index, placement or row in the input data";
    case MD_ERR_TIMEOUT: return "MD_ERR_TIMEOUT: a bounded device-side wait ran out";
    default: return "unknown md_status";
    }
}

extern "C" int md_version(void) { return 100; }

extern "C" uint64_t md_launch_count(void) { return md::g_launches.load(std::memory_order_relaxed); }

extern "C" uint64_t md_memset_count(void) { return md::g_memsets.load(std::memory_order_relaxed); }

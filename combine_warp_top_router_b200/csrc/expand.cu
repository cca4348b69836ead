// expand.cu -- receiver-side expand of deduplicated rows (md_dedup_expand).
//
// "Expert Coupling in MoE Pretraining" (PicX summary), Method 1, Deduplicating
// Dispatcher: a rank receives one row per (token, rank) that carries all of
// the token's experts on that rank.  Before the experts run, every selected
// expert needs its own copy of the row, in the conventional expert-grouped
// order (p[e], e, t) that a grouped GEMM consumes:
//     out[assign_row[t][j]] = wire[row_of_slot[t][j]]   for every slot (t, j).
//
// Rows of 1 KiB and more move by TMA bulk copies.  A unit is one slot and one
// piece (up to 4 KiB) of its row; each warp runs a ring of kStages
// shared-memory slots, loading kAhead units ahead.  The source row of a unit
// must be known before its load is issued, so the lanes of a warp fetch the
// row indices of the warp's next 32 units at once, a batch ahead, and lane 0
// reads them by shuffle.  A unit with an out-of-range source completes its
// ring slot with a plain arrive and is reported.  Slots of one token that
// share a deduplicated row load it within a few units of each other, so the
// repeats are served by L2.
// Shorter rows: one warp per slot, 16-byte vectors.
#include "common.cuh"

namespace {

constexpr int kWarps = 4;
constexpr int kStages = 4;
constexpr int kAhead = 2;
constexpr int kPiece = 4096;
constexpr int kMinRowBytes = 1024;
constexpr long long kPolls = 1ll << 22;

__global__ void __launch_bounds__(kWarps * 32)
    k_expand_tma(const char *__restrict__ wire, int64_t n_wire, int rowbytes, int pieces,
                 const int32_t *__restrict__ row_of_slot, const int32_t *__restrict__ assign_row,
                 int64_t n_slots, int64_t out_rows, char *__restrict__ out, int32_t *status,
                 long long polls, int64_t skip_unit)
{
    extern __shared__ __align__(128) unsigned char ring_all[];
    __shared__ uint64_t bars[kWarps][kStages];
    const int lane = threadIdx.x & 31, wl = threadIdx.x >> 5;
    unsigned char *ring = ring_all + (size_t)wl * kStages * kPiece;
    uint64_t *bar = bars[wl];
    const int64_t U = n_slots * pieces;
    const int64_t gw = (int64_t)blockIdx.x * kWarps + wl;
    const int64_t nw = (int64_t)gridDim.x * kWarps;
    if (lane == 0) {
        for (int st = 0; st < kStages; ++st) md::mbar_init(&bar[st], 1);
        md::fence_mbar_init();
    }
    __syncwarp();
    if (gw >= U) return;

    auto slot_of = [&](int64_t u) { return pieces == 1 ? u : u / pieces; };
    auto piece_of = [&](int64_t u) { return pieces == 1 ? 0 : (int)(u - (u / pieces) * pieces); };
    auto bytes_of = [&](int64_t u) {
        const int b = rowbytes - piece_of(u) * kPiece;
        return (uint32_t)(b < kPiece ? b : kPiece);
    };
    // lane j: source and destination rows of the warp's unit number i0 + j
    // (-1 past the end)
    auto fetch = [&](int64_t i0, int &sr, int &dr) {
        const int64_t u = gw + (i0 + lane) * nw;
        sr = -1;
        dr = -1;
        if (u < U) {
            const int64_t m = slot_of(u);
            sr = __ldg(row_of_slot + m);
            dr = __ldg(assign_row + m);
        }
    };
    int cs, cd, ns, nd;  // this batch of 32 units, and the next
    fetch(0, cs, cd);
    fetch(32, ns, nd);
    // source row of the warp's unit i, for i in this batch or the next
    auto src_at = [&](int64_t i, int64_t batch0) {
        const int j = (int)(i - batch0);
        const int a = __shfl_sync(0xffffffffu, cs, j & 31);
        const int b = __shfl_sync(0xffffffffu, ns, j & 31);
        return j < 32 ? a : b;
    };
    auto issue = [&](int64_t u, int src, int st) {
        if (u == skip_unit) return;  // test hook: this unit's slot never completes
        if (src >= 0 && src < n_wire) {
            const uint32_t nb = bytes_of(u);
            md::mbar_expect_tx(&bar[st], nb);
            md::bulk_load(ring + (size_t)st * kPiece,
                          wire + (int64_t)src * rowbytes + (int64_t)piece_of(u) * kPiece, nb, &bar[st]);
        } else {
            md::mbar_arrive(&bar[st]);
        }
    };

    for (int j = 0; j < kAhead; ++j) {
        const int sj = src_at(j, 0);
        if (lane == 0 && gw + j * nw < U) issue(gw + j * nw, sj, j % kStages);
    }
    int64_t batch0 = 0;
    int64_t i = 0;
    for (int64_t u = gw; u < U; u += nw, ++i) {
        if (i - batch0 == 32) {
            cs = ns;
            cd = nd;
            batch0 += 32;
            fetch(batch0 + 32, ns, nd);
        }
        const int st = (int)(i % kStages);
        const int64_t ua = u + (int64_t)kAhead * nw;
        const int sa = src_at(i + kAhead, batch0);
        if (lane == 0 && ua < U) {
            // the ring slot of unit i + kAhead was last read by the store of
            // unit i + kAhead - kStages
            md::bulk_wait_read<kStages - kAhead - 1>();
            issue(ua, sa, (int)((i + kAhead) % kStages));
        }
        const int j = (int)(i - batch0);
        const int src = __shfl_sync(0xffffffffu, cs, j);
        const int dst = __shfl_sync(0xffffffffu, cd, j);
        int ok = 1;
        if (lane == 0) ok = md::mbar_wait_bounded(&bar[st], (uint32_t)((i / kStages) & 1), polls);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
            md::report(status, MD_ERR_TIMEOUT);
            // wait, again bounded, for the load that timed out and the ones
            // issued after it; one late beyond both bounds can still land in
            // shared memory after the block has exited
            if (lane == 0)
                for (int a = 0; a <= kAhead; ++a)
                    if (u + a * nw < U)
                        md::mbar_wait_bounded(&bar[(i + a) % kStages],
                                              (uint32_t)(((i + a) / kStages) & 1), polls);
            break;
        }
        const bool valid = src >= 0 && src < n_wire && dst >= 0 && dst < out_rows;
        if (lane == 0) {
            if (valid)
                md::bulk_store(out + (int64_t)dst * rowbytes + (int64_t)piece_of(u) * kPiece,
                               ring + (size_t)st * kPiece, bytes_of(u));
            else if (piece_of(u) == 0)
                md::report(status, MD_ERR_DATA);
            md::bulk_commit();
        }
    }
    if (lane == 0) md::bulk_wait_all();
}

// Rows under 1 KiB: one warp per slot, 16-byte vectors.
__global__ void __launch_bounds__(256)
    k_expand_vec(const uint4 *__restrict__ wire, int64_t n_wire, int C,
                 const int32_t *__restrict__ row_of_slot, const int32_t *__restrict__ assign_row,
                 int64_t n_slots, int64_t out_rows, uint4 *__restrict__ out, int32_t *status)
{
    const int lane = threadIdx.x & 31;
    const int64_t w0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t m = w0; m < n_slots; m += nw) {
        const int src = __ldg(row_of_slot + m), dst = __ldg(assign_row + m);
        if (src < 0 || src >= n_wire || dst < 0 || dst >= out_rows) {
            if (lane == 0) md::report(status, MD_ERR_DATA);
            continue;
        }
        const uint4 *s = wire + (int64_t)src * C;
        uint4 *d = out + (int64_t)dst * C;
        for (int c = lane; c < C; c += 32) md::st_stream(d + c, md::ld_stream(s + c));
    }
}

}  // namespace

extern "C" int md_dedup_expand(const void *wire, int64_t n_wire, int H, const int32_t *row_of_slot,
                               const int32_t *assign_row, int64_t T, int k, int64_t out_rows,
                               void *out, int32_t *dev_status, void *stream)
{
    if (T < 0 || H < 8 || H % 8 != 0 || k < 1 || k > MD_MAX_TOPK || n_wire < 0 || out_rows < 0)
        return MD_ERR_ARG;
    if (T > 0 && (!row_of_slot || !assign_row)) return MD_ERR_ARG;
    if (n_wire > 0 && (!wire || !md::aligned16(wire))) return MD_ERR_ARG;
    if (out_rows > 0 && (!out || !md::aligned16(out))) return MD_ERR_ARG;
    if (T > 0 && n_wire > INT32_MAX) return MD_ERR_UNSUPPORTED;
    cudaStream_t s = md::as_stream(stream);
    int rc = md::clear_status(dev_status, s);
    if (rc != MD_OK || T == 0) return rc;
    const int64_t n_slots = T * k;
    const int rowbytes = 2 * H;
    if (rowbytes >= kMinRowBytes) {
        const int pieces = (rowbytes + kPiece - 1) / kPiece;
        const size_t smem = (size_t)kWarps * kStages * kPiece;
        static std::atomic<uint64_t> attr_done{0};
        md::once_per_device(attr_done, [smem] {
            if (cudaFuncSetAttribute(k_expand_tma, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
                cudaSuccess)
                cudaGetLastError();  // the launch then fails and reports MD_ERR_CUDA
        });
        int64_t blocks = (n_slots * pieces + kWarps - 1) / kWarps;
        if (blocks > md::sm_count()) blocks = md::sm_count();
        k_expand_tma<<<(unsigned)(blocks < 1 ? 1 : blocks), kWarps * 32, smem, s>>>(
            static_cast<const char *>(wire), n_wire, rowbytes, pieces, row_of_slot, assign_row,
            n_slots, out_rows, static_cast<char *>(out), dev_status, md::hook_poll_limit(kPolls),
            md::hook_expand_skip_unit());
    } else {
        int64_t blocks = (n_slots + 7) / 8;
        const int64_t cap = (int64_t)md::sm_count() * 8;
        if (blocks > cap) blocks = cap;
        k_expand_vec<<<(unsigned)(blocks < 1 ? 1 : blocks), 256, 0, s>>>(
            static_cast<const uint4 *>(wire), n_wire, rowbytes / 16, row_of_slot, assign_row, n_slots,
            out_rows, static_cast<uint4 *>(out), dev_status);
    }
    md::count_launches(1);
    return md::launch_status();
}

// plan_harness.cu -- host-only check of the launch planners against the
// invariants their kernels rely on.  Built and run by test_host_plans.py on
// the CPU (no GPU needed: only the host-side planning functions run).
//
// Checked for every shape of a sweep:
//   - dynamic + static shared memory of every planned launch fits a CTA
//     (227 KB), and cluster sizes stay within 8;
//   - the persistent kernels (Q1 bit-plane, INT4 M=1, small batch) have at
//     least 8 warps and their shape preconditions (K, N multiples);
//   - the Q1 and INT4 persistent kernels: replaying the kernels' own split
//     of cells into per-CTA ranges and of steps into per-warp ranges, every
//     warp's range is at least one cell long, so a cell cut between two
//     warps has exactly two parts (the kernels combine exactly two);
//   - the small-batch persistent kernel: its consumer warps and the producer
//     warp fit the launch bound, and its rounds cover every 32-row block
//     exactly once.
#include <cstdio>
#include <vector>

#include "q1_gemv_m1.cu"
#include "int4_gemv_m1.cu"
#include "gemm_smallm.cu"

using namespace lowbit;

static int g_checked = 0, g_failed = 0;
#define CHECK(cond, ...)                         \
    do {                                         \
        ++g_checked;                             \
        if (!(cond)) {                           \
            ++g_failed;                          \
            if (g_failed <= 20) {                \
                std::printf("FAIL %s: ", #cond); \
                std::printf(__VA_ARGS__);        \
                std::printf("\n");               \
            }                                    \
        }                                        \
    } while (0)

constexpr int kSms = 148;
constexpr size_t kCtaSmem = 227 * 1024;

// The persistent kernels' split: CTA b takes cells [b*C/G, (b+1)*C/G), its
// T = (c1-c0)*spc steps go to warps as [w*T/nw, (w+1)*T/nw).
static bool ranges_ok(long long cells, int grid, int nw, int spc, const char *what, int R, int N, int K)
{
    bool ok = true;
    for (int b = 0; b < grid; ++b) {
        const long long c0 = (long long)b * cells / grid, c1 = (long long)(b + 1) * cells / grid;
        const long long T = (c1 - c0) * spc;
        for (int w = 0; w < nw; ++w) {
            const long long s0 = w * T / nw, s1 = (w + 1) * T / nw;
            if (T > 0 && s1 - s0 < spc) ok = false;
        }
    }
    CHECK(ok, "%s R=%d N=%d K=%d: a warp range shorter than a cell", what, R, N, K);
    return ok;
}

int main()
{
    const int Rs[] = {1, 2, 3, 5, 8, 10, 17, 37, 64, 108, 169, 256};
    const int Ns[] = {1, 32, 64, 100, 515, 1000, 1024, 4096, 5120, 11008, 17408};
    const int Ks[] = {128, 256, 384, 1024, 1280, 2048, 3072, 4096, 5120, 11008, 17408, 32768};

    for (int R : Rs)
        for (int N : Ns)
            for (int K : Ks) {
                // --- Q1_0_g128 at M = 1 and the several-vector bit-plane forms
                for (int mv : {1, 2, 4})
                    for (bool aligned : {false, true}) {
                        const Q1Plan P = q1_plan(R, N, K, kSms, aligned, mv);
                        if (P.lean) {
                            const size_t stat = (size_t)2 * q1l_max_warps(mv) * mv * kQ1StepRows * 4;
                            CHECK(K % 1024 == 0 && N % 32 == 0, "q1 lean shape R=%d N=%d K=%d", R, N, K);
                            CHECK(P.warps >= kQ1LMinWarps && P.warps <= q1l_max_warps(mv), "q1 lean warps %d", P.warps);
                            CHECK(P.smem <= (size_t)kQ1MaxSmem && P.smem + stat <= kCtaSmem,
                                  "q1 lean smem %zu + %zu (R=%d N=%d K=%d mv=%d)", P.smem, stat, R, N, K, mv);
                            CHECK(P.act_smem == (size_t)mv * P.nchunks * (kQ1FragBytesPerChunk + kQ1InfoBytesPerChunk) +
                                                    kQ1ZeroBytes,
                                  "q1 lean activation size");
                            CHECK(P.grid_x == kSms, "q1 lean grid");
                            ranges_ok((long long)R * P.blocksN, P.grid_x, P.warps, P.nchunks / kQ1LChunks, "q1 lean", R, N,
                                      K);
                        } else if (mv == 1 && P.ok) {
                            CHECK(P.smem <= (size_t)kQ1MaxSmem, "q1 plan smem %zu (R=%d N=%d K=%d)", P.smem, R, N, K);
                            if (!P.stream) CHECK(P.nslices >= 1 && P.nslices <= kQ1MaxCluster && P.grid_y < 65536,
                                                 "q1 split slices %d", P.nslices);
                        }
                    }
                // --- INT4_G64 at M = 1: single matrix and group
                if (K % 128 == 0) {
                    const I4Plan P = i4_plan(N, K, kSms);
                    if (P.ok)
                        CHECK(P.smem <= (size_t)kI4MaxSmem && P.nslices >= 1 && P.nslices <= kI4MaxCluster,
                              "int4 split plan N=%d K=%d", N, K);
                    const I4GPlan G = i4g_plan(R, N, K, kSms);
                    if (G.ok) {
                        const size_t stat = (size_t)2 * kI4LMaxWarps * kI4StepRows * 4;
                        CHECK(N % 32 == 0, "int4 lean shape");
                        CHECK(G.warps >= kI4LMinWarps && G.warps <= kI4LMaxWarps, "int4 lean warps %d", G.warps);
                        CHECK(G.smem + stat <= kCtaSmem, "int4 lean smem %zu (R=%d N=%d K=%d)", G.smem, R, N, K);
                        ranges_ok((long long)R * G.blocksN, kSms, G.warps, G.npairs, "int4 lean", R, N, K);
                    }
                }
                // --- small batch: single matrix and group, both formats
                for (int fmt : {1, 3})
                    for (int M : {2, 3, 4, 5, 8, 9, 16, 17, 24, 32}) {
                        const SmPlan S = sm_plan(fmt, M, N, K, kSms);
                        if (S.ok)
                            CHECK(S.S >= 1 && S.S <= kSmMaxCluster && S.smem <= (size_t)kSmMaxSmem,
                                  "smallm plan fmt=%d M=%d N=%d K=%d", fmt, M, N, K);
                        const SgPlan G = sg_plan(fmt, R, M, N, K, kSms);
                        if (G.ok) {
                            CHECK(G.warps >= kSgMinWarps && G.warps <= kSgMaxWarps, "grouped smallm warps %d", G.warps);
                            CHECK(G.warps <= sg_max_warps(fmt, G.NT), "grouped smallm warps %d above the launch bound", G.warps);
                            CHECK(G.smem + 128 <= kCtaSmem && G.smem <= (size_t)kSmMaxSmem, "grouped smallm smem %zu",
                                  G.smem);
                            // round j, CTA b, warp w takes block (j*grid + b)*nw + w: all blocks, once
                            std::vector<int> seen(G.nblocks, 0);
                            for (int j = 0; j < G.rounds; ++j)
                                for (int b = 0; b < kSms; ++b)
                                    for (int w = 0; w < G.warps; ++w) {
                                        const long long blk = ((long long)j * kSms + b) * G.warps + w;
                                        if (blk < G.nblocks) ++seen[blk];
                                    }
                            bool once = true;
                            for (int v : seen) once = once && v == 1;
                            CHECK(once, "grouped smallm rounds fmt=%d R=%d M=%d N=%d K=%d", fmt, R, M, N, K);
                        }
                    }
            }
    std::printf("checked %d invariants, %d failed\n", g_checked, g_failed);
    return g_failed == 0 ? 0 : 1;
}

// stepq_host.cpp -- host-side parts of libstepq: error reporting, argument checks, the packed
// layout and the offline lifetime-aware bit allocation (STEPQuant §3.2, App. C.2).
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <limits>
#include <map>
#include <mutex>
#include <queue>
#include <utility>
#include <vector>

#include "stepq_internal.h"

namespace stepq {

static thread_local std::string g_last_error;

int set_error(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    std::vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return code;
}

void clear_error() { g_last_error.clear(); }

int check_ptrs(const char* fn, std::initializer_list<std::pair<const char*, const void*>> ptrs) {
    for (const auto& p : ptrs) {
        if (!p.second) return set_error(STEPQ_EINVAL, "%s: %s is NULL", fn, p.first);
        if (!aligned16(p.second)) return set_error(STEPQ_EALIGN, "%s: %s is not 16-byte aligned", fn, p.first);
    }
    return STEPQ_OK;
}

int check_launch(const char* fn) {
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(STEPQ_ECUDA, "%s: %s", fn, cudaGetErrorString(e));
    return STEPQ_OK;
}

int persistent_grid(const void* kernel, int threads, size_t smem, long long tiles, const char* fn, int* grid) {
    struct Entry {
        int sms = 0, per_sm = 0;
    };
    static std::mutex mu;
    static std::map<std::pair<const void*, int>, Entry> cache;   // (kernel, device)
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return set_error(STEPQ_ECUDA, "%s: %s", fn, cudaGetErrorString(e));
    Entry ent;
    {
        std::lock_guard<std::mutex> lock(mu);
        auto it = cache.find({kernel, dev});
        if (it != cache.end()) ent = it->second;
    }
    if (ent.per_sm == 0) {
        e = cudaDeviceGetAttribute(&ent.sms, cudaDevAttrMultiProcessorCount, dev);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&ent.per_sm, kernel, threads, smem);
        if (e != cudaSuccess) return set_error(STEPQ_ECUDA, "%s: %s", fn, cudaGetErrorString(e));
        if (ent.per_sm < 1) return set_error(STEPQ_ECUDA, "%s: the kernel does not fit on an SM", fn);
        std::lock_guard<std::mutex> lock(mu);
        cache[{kernel, dev}] = ent;
    }
    const long long g = static_cast<long long>(ent.sms) * ent.per_sm;
    *grid = static_cast<int>(std::min<long long>(g, std::max<long long>(tiles, 1)));
    return STEPQ_OK;
}

// ---------------------------------------------------------------------------------------------
// bit allocation
// ---------------------------------------------------------------------------------------------

// Multiple-choice DP over the units, solved from the last unit backwards so that the forward
// reconstruction can prefer the smallest candidate at every unit among equal optima.
static int allocate_dp(int n, int nc, const int* cand, const double* J, int64_t budget, uint8_t* out) {
    if (budget < 0) return set_error(STEPQ_EBUDGET, "stepq_allocate_bits: negative budget");
    const size_t W = static_cast<size_t>(budget) + 1;
    if (static_cast<double>(n + 1) * static_cast<double>(W) > 6.0e7)
        return set_error(STEPQ_EINVAL, "stepq_allocate_bits: DP table too large (%d units x %lld bits)", n,
                         (long long)budget);
    const double inf = std::numeric_limits<double>::infinity();
    std::vector<double> next(W, inf), cur(W);
    std::vector<std::vector<double>> table;   // table[u] = G_u over all bit counts
    table.reserve(static_cast<size_t>(n) + 1);
    next[0] = 0.0;
    table.push_back(next);   // G_n
    for (int u = n - 1; u >= 0; --u) {
        const double* Ju = J + static_cast<size_t>(u) * nc;
        for (size_t s = 0; s < W; ++s) {
            double best = inf;
            for (int c = 0; c < nc; ++c) {
                if (static_cast<size_t>(cand[c]) > s) break;   // ascending candidates
                const double g = next[s - cand[c]];
                if (g == inf) continue;
                best = std::min(best, Ju[c] + g);
            }
            cur[s] = best;
        }
        table.push_back(cur);
        std::swap(next, cur);
    }
    std::reverse(table.begin(), table.end());   // table[u] = G_u
    if (table[0][budget] == inf)
        return set_error(STEPQ_EBUDGET, "stepq_allocate_bits: no assignment uses exactly %lld bits", (long long)budget);
    size_t s = static_cast<size_t>(budget);
    for (int u = 0; u < n; ++u) {
        const double* Ju = J + static_cast<size_t>(u) * nc;
        for (int c = 0; c < nc; ++c) {
            if (static_cast<size_t>(cand[c]) > s) break;
            const double g = table[u + 1][s - cand[c]];
            if (g != inf && Ju[c] + g == table[u][s]) {
                out[u] = static_cast<uint8_t>(cand[c]);
                s -= cand[c];
                break;
            }
        }
    }
    return STEPQ_OK;
}

// Lagrangian allocation: walk every unit along the lower convex hull of (cand, J) in order of
// the steepest objective decrease per bit, then repair the remainder exactly.
static int allocate_lagrange(int n, int nc, const int* cand, const double* J, int64_t budget, uint8_t* out) {
    std::vector<std::vector<int>> hull(n);
    std::vector<int> at(n, 0), pick(n);
    int64_t used = 0;
    for (int u = 0; u < n; ++u) {
        const double* Ju = J + static_cast<size_t>(u) * nc;
        auto& hu = hull[u];
        for (int c = 0; c < nc; ++c) {
            while (hu.size() >= 2) {
                const int a = hu[hu.size() - 2], b = hu.back();
                const double left = (Ju[b] - Ju[a]) / static_cast<double>(cand[b] - cand[a]);
                const double right = (Ju[c] - Ju[b]) / static_cast<double>(cand[c] - cand[b]);
                if (left >= right) hu.pop_back();
                else break;
            }
            hu.push_back(c);
        }
        pick[u] = hu[0];
        used += cand[hu[0]];
    }
    int64_t rem = budget - used;
    if (rem < 0)
        return set_error(STEPQ_EBUDGET, "stepq_allocate_bits: budget %lld below the smallest widths",
                         (long long)budget);

    // (slope, unit), smallest slope first, then lowest unit.
    using Move = std::pair<double, int>;
    std::priority_queue<Move, std::vector<Move>, std::greater<Move>> heap;
    auto push_next = [&](int u) {
        const auto& hu = hull[u];
        if (at[u] + 1 >= static_cast<int>(hu.size())) return;
        const int a = hu[at[u]], b = hu[at[u] + 1];
        const double* Ju = J + static_cast<size_t>(u) * nc;
        heap.emplace((Ju[b] - Ju[a]) / static_cast<double>(cand[b] - cand[a]), u);
    };
    for (int u = 0; u < n; ++u) push_next(u);
    while (!heap.empty()) {
        const int u = heap.top().second;
        heap.pop();
        const int a = hull[u][at[u]], b = hull[u][at[u] + 1];
        const int64_t db = cand[b] - cand[a];
        if (db > rem) continue;   // never fits again: the remainder only shrinks
        rem -= db;
        at[u] += 1;
        pick[u] = b;
        push_next(u);
    }

    if (rem > 0) {
        // Repair: the least change of J that reaches the budget exactly, singles before pairs,
        // then lowest (u, v, new width of u, new width of v).
        bool found = false;
        double best = 0.0;
        int bu = -1, bku = -1, bv = -1, bkv = -1;
        for (int u = 0; u < n; ++u) {
            const double* Ju = J + static_cast<size_t>(u) * nc;
            for (int c = 0; c < nc; ++c) {
                if (cand[c] - cand[pick[u]] != rem) continue;
                const double dj = Ju[c] - Ju[pick[u]];
                if (!found || dj < best) { found = true; best = dj; bu = u; bku = c; bv = -1; }
            }
        }
        // Lowest and second-lowest down-move change per size, to bound each (u, up-move).
        const double inf = std::numeric_limits<double>::infinity();
        const int maxd = cand[nc - 1] - cand[0];
        std::vector<double> min1(maxd + 1, inf), min2(maxd + 1, inf);
        std::vector<int> arg1(maxd + 1, -1);
        for (int v = 0; v < n; ++v) {
            const double* Jv = J + static_cast<size_t>(v) * nc;
            for (int c = 0; c < nc; ++c) {
                const int d = cand[pick[v]] - cand[c];
                if (d <= 0) continue;
                const double dj = Jv[c] - Jv[pick[v]];
                if (dj < min1[d]) {
                    if (arg1[d] != v) min2[d] = min1[d];
                    min1[d] = dj;
                    arg1[d] = v;
                } else if (v != arg1[d] && dj < min2[d]) {
                    min2[d] = dj;
                }
            }
        }
        for (int u = 0; u < n; ++u) {
            const double* Ju = J + static_cast<size_t>(u) * nc;
            for (int cu = 0; cu < nc; ++cu) {
                const int64_t up = cand[cu] - cand[pick[u]];
                if (up <= 0) continue;
                const int64_t down = up - rem;
                if (down <= 0 || down > maxd) continue;
                const double A = Ju[cu] - Ju[pick[u]];
                const double bound_b = (arg1[down] == u) ? min2[down] : min1[down];
                if (bound_b == inf) continue;
                if (found && A + bound_b >= best) continue;   // cannot be strictly better
                for (int v = 0; v < n; ++v) {
                    if (v == u) continue;
                    const double* Jv = J + static_cast<size_t>(v) * nc;
                    for (int cv = 0; cv < nc; ++cv) {
                        if (cand[pick[v]] - cand[cv] != down) continue;
                        const double dj = A + (Jv[cv] - Jv[pick[v]]);
                        if (!found || dj < best) { found = true; best = dj; bu = u; bku = cu; bv = v; bkv = cv; }
                    }
                }
            }
        }
        if (!found)
            return set_error(STEPQ_EBUDGET, "stepq_allocate_bits: no move reaches the budget (%lld bits left)",
                             (long long)rem);
        pick[bu] = bku;
        if (bv >= 0) pick[bv] = bkv;
    }
    for (int u = 0; u < n; ++u) out[u] = static_cast<uint8_t>(cand[pick[u]]);
    return STEPQ_OK;
}

}  // namespace stepq

using namespace stepq;

extern "C" const char* stepq_last_error(void) { return g_last_error.c_str(); }

extern "C" const char* stepq_build_info(void) {
    return "libstepq: STEPQuant quantized gated Delta-rule decode; sm_100a; d in {64,128}; widths {2,4,6,8} and FP16 pivot rows (16)";
}

extern "C" int stepq_packed_layout(stepq_dims dims, const uint8_t* bits_host, int64_t* head_off_host,
                                   int64_t* bytes_per_seq, int64_t* total_bytes) {
    clear_error();
    int rc = check_dims(dims, "stepq_packed_layout");
    if (rc) return rc;
    if (!bits_host) return set_error(STEPQ_EINVAL, "stepq_packed_layout: bits_host is NULL");
    int64_t off = 0;
    for (int h = 0; h < dims.H; ++h) {
        if (head_off_host) head_off_host[h] = off;
        int64_t sum = 0;
        for (int i = 0; i < dims.dk; ++i) {
            const int b = bits_host[static_cast<int64_t>(h) * dims.dk + i];
            if (b != 2 && b != 4 && b != 6 && b != 8 && b != 16)
                return set_error(STEPQ_EUNSUPPORTED, "stepq_packed_layout: bits[%d][%d] = %d", h, i, b);
            sum += b;
        }
        off += sum * (dims.dv / 8);
    }
    if (bytes_per_seq) *bytes_per_seq = off;
    if (total_bytes) *total_bytes = off * static_cast<int64_t>(dims.B);
    return STEPQ_OK;
}

extern "C" int stepq_allocate_bits(int n_units, int n_cand, const int* cand_host, const double* J_host,
                                   int64_t budget_bits, int mode, uint8_t* bits_out_host) {
    clear_error();
    if (n_units <= 0 || n_cand <= 0 || !cand_host || !J_host || !bits_out_host)
        return set_error(STEPQ_EINVAL, "stepq_allocate_bits: n_units=%d n_cand=%d", n_units, n_cand);
    for (int c = 0; c < n_cand; ++c) {
        if (cand_host[c] <= 0 || cand_host[c] > 16 || (c > 0 && cand_host[c] <= cand_host[c - 1]))
            return set_error(STEPQ_EINVAL, "stepq_allocate_bits: candidates must ascend within 1..16");
    }
    for (int64_t e = 0; e < static_cast<int64_t>(n_units) * n_cand; ++e)
        if (!std::isfinite(J_host[e])) return set_error(STEPQ_EINVAL, "stepq_allocate_bits: J[%lld] not finite", (long long)e);
    if (mode == 1) return allocate_dp(n_units, n_cand, cand_host, J_host, budget_bits, bits_out_host);
    if (mode == 0) return allocate_lagrange(n_units, n_cand, cand_host, J_host, budget_bits, bits_out_host);
    return set_error(STEPQ_EINVAL, "stepq_allocate_bits: mode %d", mode);
}

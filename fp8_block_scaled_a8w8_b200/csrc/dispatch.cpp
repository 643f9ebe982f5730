// Dispatch table: rows keyed (op, padded M, N, K) naming a kernel configuration,
// the padded-M lookup walk, and the lookup census.
//
// Walk ([aiter#7752] "[Perf] Retune gfx942 Qwen3.8-27B a8w8 blockscale decode rows
// for cold weights", section "PR-specific question"): probe exact M; then the next
// power of two if M < 16, or the next multiple of 16 if 16 <= M <= 256; then the next
// power of two; else miss. [cookbook#8] "Two amplifiers": M = 6016 therefore runs the
// row tuned for 8192. A miss runs the per-shape default configuration
// ([mi210 docs/43] section 6: a miss returns None and the default kernel runs).
// Census ([cookbook#8], coverage_report.py review): lookups are counted per distinct
// key so duplicates collapse.
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <tuple>
#include <vector>

#include "internal.h"

namespace fp8bs {

// ------------------------------------------------------------ configurations
static const KernelConfig kConfigs[] = {
    // name                    op                          path       bn  sk  depth
    {"a8w8_gemv_d2", FP8BS_OP_A8W8_BLOCKSCALE, kPathGemv, 0, 1, 2},
    {"a8w8_gemv_d3", FP8BS_OP_A8W8_BLOCKSCALE, kPathGemv, 0, 1, 3},
    {"a8w8_gemv_d4", FP8BS_OP_A8W8_BLOCKSCALE, kPathGemv, 0, 1, 4},
    {"a8w8_gemv_tma", FP8BS_OP_A8W8_BLOCKSCALE, kPathGemvTma, 0, 1, 0},
    {"a8w8_gemv_umma", FP8BS_OP_A8W8_BLOCKSCALE, kPathGemvUmma, 0, 1, 0},
    {"a8w8_tc_bn128", FP8BS_OP_A8W8_BLOCKSCALE, kPathTc, 128, 0, 0},
    {"a8w8_tc_bn256", FP8BS_OP_A8W8_BLOCKSCALE, kPathTc, 256, 0, 0},
    {"a8w8_tcw_bn128", FP8BS_OP_A8W8_BLOCKSCALE, kPathTcWide, 128, 0, 0},
    {"a8w8_tcw_bn256", FP8BS_OP_A8W8_BLOCKSCALE, kPathTcWide, 256, 0, 0},
    // fixed K splits for the tuner (mid M, where the tiles leave SMs idle)
    {"a8w8_tcw_bn128_sk2", FP8BS_OP_A8W8_BLOCKSCALE, kPathTcWide, 128, 2, 0},
    {"a8w8_tcw_bn128_sk4", FP8BS_OP_A8W8_BLOCKSCALE, kPathTcWide, 128, 4, 0},
    {"a8w8_tcw_bn128_sk6", FP8BS_OP_A8W8_BLOCKSCALE, kPathTcWide, 128, 6, 0},
    {"a8w8_tcw_bn128_sk8", FP8BS_OP_A8W8_BLOCKSCALE, kPathTcWide, 128, 8, 0},
    {"a8w8_tcw_bn256_sk2", FP8BS_OP_A8W8_BLOCKSCALE, kPathTcWide, 256, 2, 0},
    {"a8w8_tcw_bn256_sk4", FP8BS_OP_A8W8_BLOCKSCALE, kPathTcWide, 256, 4, 0},
    {"a8w8_tc2_bn256", FP8BS_OP_A8W8_BLOCKSCALE, kPathTcPair, 256, 1, 1},   // depth: MMA halves per K step
    {"a8w8_tc2h_bn256", FP8BS_OP_A8W8_BLOCKSCALE, kPathTcPair, 256, 1, 2},
    {"bf16_gemv_d2", FP8BS_OP_BF16, kPathGemv, 0, 1, 2},
    {"bf16_gemv_d4", FP8BS_OP_BF16, kPathGemv, 0, 1, 4},
    {"bf16_gemv_umma", FP8BS_OP_BF16, kPathGemvUmma, 0, 1, 0},
    {"bf16_tc_bn32", FP8BS_OP_BF16, kPathTc, 32, 0, 0},
    {"bf16_tc_bn64", FP8BS_OP_BF16, kPathTc, 64, 0, 0},
    {"bf16_tc_bn128", FP8BS_OP_BF16, kPathTc, 128, 0, 0},
    {"bf16_tc_bn192", FP8BS_OP_BF16, kPathTc, 192, 0, 0},
    {"bf16_tc_bn256", FP8BS_OP_BF16, kPathTc, 256, 0, 0},
};
static constexpr int kNumConfigs = sizeof(kConfigs) / sizeof(kConfigs[0]);

const KernelConfig* find_config(int op, const char* name) {
  if (!name) return nullptr;
  for (const auto& c : kConfigs)
    if (c.op == op && std::strcmp(c.name, name) == 0) return &c;
  return nullptr;
}

const KernelConfig* const* list_configs(int op, int* count) {
  static const KernelConfig* lists[FP8BS_NUM_OPS][kNumConfigs];
  static int counts[FP8BS_NUM_OPS];
  static std::once_flag once;
  std::call_once(once, [] {
    for (const auto& c : kConfigs) lists[c.op][counts[c.op]++] = &c;
  });
  *count = counts[op];
  return lists[op];
}

// Tensor-core tile width: the widest candidate (fewest re-reads of A) whose output tiles
// still give at least half of the SMs a tile; if none does, the narrowest (the kernel then
// also splits K).
static int pick_bn(int64_t M, int64_t N, const int* cands, int n) {
  const int64_t m_tiles = (M + 127) / 128;
  const int64_t half_sms = (int64_t(device_sm_count()) + 1) / 2;
  for (int i = 0; i < n; ++i)
    if (m_tiles * ((N + cands[i] - 1) / cands[i]) >= half_sms) return cands[i];
  return cands[n - 1];
}

const KernelConfig* default_config(int op, int64_t M, int64_t N, int64_t K) {
  (void)K;
  char nm[32];
  if (op == FP8BS_OP_A8W8_BLOCKSCALE) {
    if (M <= kGemvMaxM) return find_config(op, "a8w8_gemv_umma");
    // (the CTA-pair configurations a8w8_tc2*_bn256 measured no faster than single CTAs
    // with 128 x 256 tiles on the prefill shapes, so they are opt-in table rows)
    static const int fp8_bn[] = {256, 128};
    const int bn = (N % 256 == 0) ? pick_bn(M, N, fp8_bn, 2) : 128;
    std::snprintf(nm, sizeof nm, "a8w8_tcw_bn%d", bn);
    return find_config(op, nm);
  }
  if (M <= kGemvMaxM) return find_config(op, "bf16_gemv_umma");
  // widest first among the widths that tile N without a ragged last tile, then narrower;
  // a large N (an lm_head) takes 256 or 128 even with a ragged last tile, which costs
  // less than re-reading A for every narrow tile
  static const int all_bn[] = {256, 192, 128, 64, 32};
  int cands[5], n = 0;
  if (N >= 2048) {
    cands[n++] = 256;
    cands[n++] = 128;
  } else {
    for (int b : all_bn)
      if (b <= N && N % b == 0) cands[n++] = b;
  }
  if (n == 0) cands[n++] = 32;
  if (N < 256 && N % 32 == 0 && N != cands[0]) {  // a single tile as wide as N comes first
    for (int i = n; i > 0; --i) cands[i] = cands[i - 1];
    cands[0] = int(N);
    ++n;
  }
  int bn = pick_bn(M, N, cands, n);
  if (bn != 32 && bn != 64 && bn != 128 && bn != 192 && bn != 256) bn = 32;
  std::snprintf(nm, sizeof nm, "bf16_tc_bn%d", bn);
  return find_config(op, nm);
}

// ------------------------------------------------------------ table + census
namespace {

using Key = std::tuple<int, int64_t, int64_t, int64_t>;                        // op, M, N, K
using CensusKey = std::tuple<int, int64_t, int64_t, int64_t, int64_t, std::string>;  // op, M, N, K, padded_M, cfg

struct State {
  std::mutex mu;
  std::map<Key, const KernelConfig*> rows;
  std::map<Key, bool> tuned;  // rows whose configuration was chosen by measurement
  std::map<CensusKey, uint64_t> census;
  uint64_t hits[FP8BS_NUM_OPS] = {0, 0};
  uint64_t misses[FP8BS_NUM_OPS] = {0, 0};
  bool log = false;
};

// Rows chosen by measurement (written by the package's tune.py on a B200): each names the
// fastest configuration among those that run the shape, timed on cold weights.
struct TunedRow {
  int op;
  int64_t M, N, K;
  const char* cfg;
};
static const TunedRow kTunedRows[] = {
#include "tuned_rows.inc"
    {0, 0, 0, 0, nullptr},  // end
};

void add_builtin_rows(std::map<Key, const KernelConfig*>& rows, std::map<Key, bool>& tuned) {
  // Rows for the decode / prefill projections at the tuner's M ladder: powers of two,
  // multiples of 16 up to 256. Each carries the measured choice where the tuner has
  // timed the shape, else the default heuristic.
  const int64_t nk[][2] = {{5120, 6144}, {14336, 5120}, {16384, 5120}, {34816, 5120}};
  std::vector<int64_t> ms = {1, 2, 4, 8};
  for (int64_t m = 16; m <= 256; m += 16) ms.push_back(m);
  for (int64_t m = 512; m <= 8192; m *= 2) ms.push_back(m);
  for (const auto& p : nk)
    for (int64_t m : ms)
      rows[Key{FP8BS_OP_A8W8_BLOCKSCALE, m, p[0], p[1]}] = default_config(FP8BS_OP_A8W8_BLOCKSCALE, m, p[0], p[1]);
  const int64_t bnk[][2] = {{256, 6144}, {32, 6144}, {384, 5120}, {1024, 5120}, {128, 512}};
  const int64_t bms[] = {1, 32, 576, 4096, 16384};
  for (const auto& p : bnk)
    for (int64_t m : bms) rows[Key{FP8BS_OP_BF16, m, p[0], p[1]}] = default_config(FP8BS_OP_BF16, m, p[0], p[1]);
  for (int64_t m : {32, 512, 1024, 2048, 4096})  // lm_head (N = 32320, K = 5120) at the power-of-two ladder
    rows[Key{FP8BS_OP_BF16, m, 32320, 5120}] = default_config(FP8BS_OP_BF16, m, 32320, 5120);
  for (const auto& r : kTunedRows) {
    if (!r.cfg) continue;
    if (const KernelConfig* c = find_config(r.op, r.cfg)) {
      rows[Key{r.op, r.M, r.N, r.K}] = c;
      tuned[Key{r.op, r.M, r.N, r.K}] = true;
    }
  }
}

State& state() {
  static State* s = [] {
    auto* st = new State();
    add_builtin_rows(st->rows, st->tuned);
    const char* e = std::getenv("FP8BS_LOG_DISPATCH");
    st->log = e && e[0] == '1';
    return st;
  }();
  return *s;
}

int64_t next_pow2(int64_t m) {
  int64_t p = 1;
  while (p < m) p <<= 1;
  return p;
}

}  // namespace

const KernelConfig* dispatch(int op, int64_t M, int64_t N, int64_t K, bool record, int64_t* padded_M, bool* hit) {
  State& st = state();
  int64_t probes[3];
  int np = 0;
  probes[np++] = M;
  if (M < 16)
    probes[np++] = next_pow2(M);
  else if (M <= 256)
    probes[np++] = (M + 15) / 16 * 16;
  probes[np++] = next_pow2(M);

  std::lock_guard<std::mutex> lk(st.mu);
  const KernelConfig* cfg = nullptr;
  int64_t pm = 0;
  for (int i = 0; i < np && !cfg; ++i) {
    auto it = st.rows.find(Key{op, probes[i], N, K});
    if (it != st.rows.end()) {
      cfg = it->second;
      pm = probes[i];
    }
  }
  const bool is_hit = cfg != nullptr;
  if (!cfg) cfg = default_config(op, M, N, K);
  if (padded_M) *padded_M = pm;
  if (hit) *hit = is_hit;
  if (record && cfg) {
    (is_hit ? st.hits : st.misses)[op]++;
    auto& cnt = st.census[CensusKey{op, M, N, K, pm, cfg->name}];
    if (cnt++ == 0 && st.log)
      std::fprintf(stderr, "[fp8bs] lookup op=%d M=%lld N=%lld K=%lld padded_M=%lld %s cfg=%s\n", op,
                   (long long)M, (long long)N, (long long)K, (long long)pm, is_hit ? "hit" : "miss", cfg->name);
  }
  return cfg;
}

}  // namespace fp8bs

using namespace fp8bs;

extern "C" {

__attribute__((visibility("default"))) fp8bs_status fp8bs_dispatch_lookup(int op, int64_t M, int64_t N, int64_t K,
                                                                          int record, int64_t* padded_M, int* hit,
                                                                          char* cfg, size_t cfg_len) {
  if (op < 0 || op >= FP8BS_NUM_OPS || M <= 0 || N <= 0 || K <= 0) return FP8BS_ERR_INVALID_ARG;
  bool h = false;
  int64_t pm = 0;
  const KernelConfig* c = dispatch(op, M, N, K, record != 0, &pm, &h);
  if (!c) return FP8BS_ERR_UNSUPPORTED;
  if (padded_M) *padded_M = pm;
  if (hit) *hit = h ? 1 : 0;
  if (cfg && cfg_len) {
    std::strncpy(cfg, c->name, cfg_len - 1);
    cfg[cfg_len - 1] = 0;
  }
  return FP8BS_OK;
}

__attribute__((visibility("default"))) fp8bs_status fp8bs_dispatch_set_row(int op, int64_t M, int64_t N, int64_t K,
                                                                           const char* cfg) {
  if (op < 0 || op >= FP8BS_NUM_OPS || M <= 0 || N <= 0 || K <= 0 || !cfg) return FP8BS_ERR_INVALID_ARG;
  const KernelConfig* c = find_config(op, cfg);
  if (!c) return FP8BS_ERR_INVALID_ARG;
  if ((c->path == kPathGemv || c->path == kPathGemvTma || c->path == kPathGemvUmma) && M > kGemvMaxM)
    return FP8BS_ERR_UNSUPPORTED;
  State& st = state();
  std::lock_guard<std::mutex> lk(st.mu);
  st.rows[Key{op, M, N, K}] = c;
  st.tuned.erase(Key{op, M, N, K});
  return FP8BS_OK;
}

__attribute__((visibility("default"))) fp8bs_status fp8bs_dispatch_reset_table(int keep_builtin) {
  State& st = state();
  std::lock_guard<std::mutex> lk(st.mu);
  st.rows.clear();
  st.tuned.clear();
  if (keep_builtin) add_builtin_rows(st.rows, st.tuned);
  return FP8BS_OK;
}

__attribute__((visibility("default"))) fp8bs_status fp8bs_dispatch_list_configs(int op, char* buf, size_t len) {
  if (op < 0 || op >= FP8BS_NUM_OPS || !buf || !len) return FP8BS_ERR_INVALID_ARG;
  int n = 0;
  const KernelConfig* const* l = list_configs(op, &n);
  std::string s;
  for (int i = 0; i < n; ++i) {
    s += l[i]->name;
    s += '\n';
  }
  std::strncpy(buf, s.c_str(), len - 1);
  buf[len - 1] = 0;
  return s.size() < len ? FP8BS_OK : FP8BS_ERR_INVALID_ARG;
}

__attribute__((visibility("default"))) fp8bs_status fp8bs_dispatch_stats(int op, uint64_t* hits, uint64_t* misses,
                                                                         uint64_t* distinct_hits,
                                                                         uint64_t* distinct_misses) {
  if (op < 0 || op >= FP8BS_NUM_OPS) return FP8BS_ERR_INVALID_ARG;
  State& st = state();
  std::lock_guard<std::mutex> lk(st.mu);
  uint64_t dh = 0, dm = 0;
  for (const auto& kv : st.census) {
    if (std::get<0>(kv.first) != op) continue;
    (std::get<4>(kv.first) != 0 ? dh : dm)++;
  }
  if (hits) *hits = st.hits[op];
  if (misses) *misses = st.misses[op];
  if (distinct_hits) *distinct_hits = dh;
  if (distinct_misses) *distinct_misses = dm;
  return FP8BS_OK;
}

__attribute__((visibility("default"))) fp8bs_status fp8bs_dispatch_reset_stats(void) {
  State& st = state();
  std::lock_guard<std::mutex> lk(st.mu);
  st.census.clear();
  for (int i = 0; i < FP8BS_NUM_OPS; ++i) st.hits[i] = st.misses[i] = 0;
  return FP8BS_OK;
}

__attribute__((visibility("default"))) fp8bs_status fp8bs_dispatch_dump_json(char* buf, size_t len) {
  if (!buf || !len) return FP8BS_ERR_INVALID_ARG;
  State& st = state();
  std::string s = "[";
  {
    std::lock_guard<std::mutex> lk(st.mu);
    bool first = true;
    char line[256];
    for (const auto& kv : st.census) {
      const auto& k = kv.first;
      std::snprintf(line, sizeof line,
                    "%s{\"op\":%d,\"M\":%lld,\"N\":%lld,\"K\":%lld,\"padded_M\":%lld,\"hit\":%s,\"cfg\":\"%s\","
                    "\"count\":%llu}",
                    first ? "" : ",", std::get<0>(k), (long long)std::get<1>(k), (long long)std::get<2>(k),
                    (long long)std::get<3>(k), (long long)std::get<4>(k), std::get<4>(k) ? "true" : "false",
                    std::get<5>(k).c_str(), (unsigned long long)kv.second);
      s += line;
      first = false;
    }
  }
  s += "]";
  if (s.size() >= len) {
    buf[0] = 0;
    return FP8BS_ERR_INVALID_ARG;
  }
  std::memcpy(buf, s.c_str(), s.size() + 1);
  return FP8BS_OK;
}

__attribute__((visibility("default"))) fp8bs_status fp8bs_dispatch_dump_table_json(char* buf, size_t len) {
  if (!buf || !len) return FP8BS_ERR_INVALID_ARG;
  State& st = state();
  std::string s = "[";
  {
    std::lock_guard<std::mutex> lk(st.mu);
    bool first = true;
    char line[256];
    for (const auto& kv : st.rows) {
      const auto& k = kv.first;
      std::snprintf(line, sizeof line, "%s{\"op\":%d,\"M\":%lld,\"N\":%lld,\"K\":%lld,\"cfg\":\"%s\",\"tuned\":%s}",
                    first ? "" : ",", std::get<0>(k), (long long)std::get<1>(k), (long long)std::get<2>(k),
                    (long long)std::get<3>(k), kv.second->name, st.tuned.count(k) ? "true" : "false");
      s += line;
      first = false;
    }
  }
  s += "]";
  if (s.size() >= len) {
    buf[0] = 0;
    return FP8BS_ERR_INVALID_ARG;
  }
  std::memcpy(buf, s.c_str(), s.size() + 1);
  return FP8BS_OK;
}

__attribute__((visibility("default"))) uint64_t fp8bs_dispatch_table_hash(void) {
  State& st = state();
  std::lock_guard<std::mutex> lk(st.mu);
  uint64_t h = 1469598103934665603ull;
  auto mix = [&h](const void* p, size_t n) {
    const unsigned char* b = static_cast<const unsigned char*>(p);
    for (size_t i = 0; i < n; ++i) {
      h ^= b[i];
      h *= 1099511628211ull;
    }
  };
  for (const auto& kv : st.rows) {
    int op = std::get<0>(kv.first);
    int64_t v[3] = {std::get<1>(kv.first), std::get<2>(kv.first), std::get<3>(kv.first)};
    mix(&op, sizeof op);
    mix(v, sizeof v);
    mix(kv.second->name, std::strlen(kv.second->name));
  }
  return h;
}

}  // extern "C"

// mk_host.cpp -- host side of the C ABI: config checks, task-graph lowering and validation,
// weight packing, arena layout, launches.
//
// Lowering follows Part 1 "Compilateur" of the MPK summary ("Compiler des LLM en MegaKernel
// ..."): every op of the decode step becomes per-SM tile tasks, edges follow the actual data
// each tile reads (attention of KV head g waits only for the QKV tiles of head group g), and
// events carry thresholds equal to their producer counts.  Queues are static and in one
// global topological order (the precomputed schedule of "Ada-MK ...", section 2, "offline
// DAG search -> fixed schedule"), which is what lets the producer warp prefetch the next
// task's weights before its inputs exist.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <string>
#include <vector>

#include "mk_internal.h"

using namespace mk;

namespace {

thread_local std::string g_err;

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct TaskRec {  // host-side task with its SM
  Task t;
  int sm;
};

struct Graph {
  std::vector<TaskRec> tasks;  // in queue order, grouped by SM (SM 0 first)
  std::vector<uint32_t> ev_count;
  int n_sms = 0;
};

}  // namespace

struct mk_ctx {
  mk_config cfg;
  int device = -1;
  int n_sms = 148;
  int variant = -1;
  int G = 1, rows_qkv = 0, rows_gu = 0, nch = 1, n_lm = 0;
  int nseg_h = 0, rps_h = 0, nseg_f = 0, rps_f = 0;
  int bm = 1;              // batch width of the decode kernel (1, or 4 with masking)
  int kdc = 0, ndc = 1;    // down-projection K chunk and chunk count (ndc > 1 when bm > 1)
  int task_rows = kTaskRows;  // rows per GEMV task (kTaskRows / bm); tensor-core: K units per task
  // tensor-core projection tiles (max_batch > 4): weights in kTcRows x kTcUnitK blocks
  bool tc = false;
  int tc_nk[8] = {0}, tc_tiles[8] = {0}, tc_tile_base[8] = {0};  // per task kind
  int n_tile_ids = 0;         // tiles of one layer's projections plus the LM head's
  size_t rec_cap = 0, n_recs = 0;  // partial records (workspace capacity, in use)
  // events
  int n_events = 0, ev_lm = 0, ev_tok = 0;
  Graph g;
  std::vector<uint32_t> qbegin;
  // arena layout
  std::vector<LayerOff> loff;
  uint64_t off_embed = 0, off_lm = 0, off_fnorm = 0, arena_bytes = 0;
  // workspace layout
  size_t ws_tasks = 0, ws_qbegin = 0, ws_evcount = 0, ws_ev = 0, ws_acnt = 0, ws_err = 0, ws_loff = 0, ws_rope = 0,
         ws_xin = 0, ws_xmid = 0, ws_q = 0, ws_o = 0, ws_h = 0, ws_part = 0, ws_lmval = 0, ws_lmidx = 0,
         ws_pf = 0, ws_tpart = 0, ws_tcnt = 0, ws_kraw = 0, ws_pools = 0, ws_pcnt = 0, ws_bytes = 0;
  size_t ev_bytes = 0, acnt_bytes = 0, tcnt_bytes = 0, pcnt_bytes = 0;
  // run-time claims (mk_set_dispatch): 0 = static queues; 1 = every projection of every layer
  // is a pool of n_sms * dyn_split tasks claimed at run time; 2 = the same, claims paced by
  // the SM's workers
  int dyn = 0, dyn_split = 2;
  std::vector<uint32_t> pool_first, pool_count;  // per pool: first task index, task count
  int pool_cap = 0;
  int pf_rows = 0;
  size_t kv_bytes = 0;
  uint64_t weight_bytes_per_step = 0;
  // runtime
  uint8_t* arena = nullptr;
  uint8_t* ws = nullptr;
  bool loaded = false;
  int B = 0;
  std::vector<int> pos;
  uint32_t epoch = 0;
  uint64_t timeout_ns = 2000000000ull;
  int drop_event = -1;
  uint64_t* trace = nullptr;
  int l2_ahead = 8;  // L2 lookahead stages while the ring is full (mk_set_l2_prefetch)
  int min_chunk_keys = kMinChunkKeysDefault;  // split-KV chunk length floor (mk_set_attn_chunk_keys)
  int head_keys = kHeadKeysDefault;           // head-mode attention up to this length (mk_set_attn_head_keys)
  std::vector<double> sm_weights;  // relative streaming speed per SM (partition weights)
  std::vector<double> op_weights[8];  // per projection kind; empty = sm_weights
  size_t task_cap = 0, lm_cap = 0; // workspace capacity for re-partitioned graphs
  std::string err;
  // Tensor parallel.  A shard context (tp_ranks > 1, no tp_shards) is rank tp_rank's part of
  // the model: 1/tp_ranks of the query and KV heads, of the ffn rows and of the vocabulary,
  // the whole hidden size.  An emulated tensor-parallel context (tp_shards non-empty) hosts
  // every rank's shard on one device in one launch; it owns the shards.
  int tp_ranks = 1, tp_rank = 0;
  int tp_vbase = 0, tp_vfull = 0;   // shard: first vocab row of the LM-head slice; full vocab
  int ev_lmx = -1;                  // shard: the argmax-exchange event
  size_t ws_recv_o = 0, ws_recv_d = 0, ws_lmx = 0, recv_o_bytes = 0;
  std::vector<mk_ctx*> tp_shards;
  int tp_sms = 0;                   // emulated: SMs per rank
  std::vector<size_t> tp_arena_off, tp_ws_off, tp_kv_off;
  size_t tp_ws_tasks = 0, tp_ws_qbegin = 0;  // emulated: the combined queues
  std::vector<Task> tp_tasks;       // emulated: every rank's tasks, rank 0's SMs first
  std::vector<int> tp_task_sm;      // their (global) SMs
  std::vector<uint32_t> tp_qbegin;
  ~mk_ctx() {
    for (mk_ctx* sh : tp_shards) delete sh;
  }
};

namespace {

int fail(mk_ctx* c, int code, const std::string& msg) {
  if (c) c->err = msg;
  g_err = msg;
  return code;
}

int pow2_floor(int x) {
  int p = 1;
  while (p * 2 <= x) p *= 2;
  return p;
}

// ---------------------------------------------------------------------------------------
// Event ids
int ev_embed() { return 0; }
int ev_base(const mk_ctx* c, int l) { return 1 + l * (c->cfg.n_kv_heads + 4); }
int ev_qkv(const mk_ctx* c, int l, int g) { return ev_base(c, l) + g; }
int ev_attn(const mk_ctx* c, int l) { return ev_base(c, l) + c->cfg.n_kv_heads; }
int ev_o(const mk_ctx* c, int l) { return ev_base(c, l) + c->cfg.n_kv_heads + 1; }
int ev_gu(const mk_ctx* c, int l) { return ev_base(c, l) + c->cfg.n_kv_heads + 2; }
int ev_down(const mk_ctx* c, int l) { return ev_base(c, l) + c->cfg.n_kv_heads + 3; }

// Split `total` rows over the SMs in contiguous ranges (multiples of gran) proportional to
// the per-SM weights (equal weights: balanced), and each range into tasks of at most
// kTaskRows rows.
std::vector<std::vector<std::pair<int, int>>> partition_rows(int total, int gran, const std::vector<double>& w,
                                                             int max_rows) {
  const int n_sms = (int)w.size();
  std::vector<std::vector<std::pair<int, int>>> out(n_sms);
  std::vector<double> cum(n_sms + 1, 0.0);
  for (int s = 0; s < n_sms; ++s) cum[s + 1] = cum[s] + w[s];
  auto bound = [&](int s) -> int {
    if (s == n_sms) return total;
    return (int)((long long)std::llround((double)total * cum[s] / cum[n_sms]) / gran * gran);
  };
  for (int s = 0; s < n_sms; ++s) {
    int a = bound(s);
    int b = bound(s + 1);
    int n = b - a;
    if (n <= 0) continue;
    int nt = (n + max_rows - 1) / max_rows;
    for (;;) {
      bool ok = true;
      std::vector<std::pair<int, int>> parts;
      for (int i = 0; i < nt; ++i) {
        int lo = (int)(((long long)n * i / nt) / gran * gran);
        int hi = (i + 1 == nt) ? n : (int)(((long long)n * (i + 1) / nt) / gran * gran);
        if (hi - lo > max_rows) ok = false;
        if (hi > lo) parts.push_back({a + lo, hi - lo});
      }
      if (ok) {
        out[s] = parts;
        break;
      }
      ++nt;
    }
  }
  return out;
}

// Tensor-core ops: the op's blocks (tile-major, K unit minor) split over the SMs in
// contiguous ranges proportional to the per-SM weights; each range cut into tasks at tile
// boundaries and after kTcUnitsMax units.  Returns per SM the (first block, blocks) pairs.
std::vector<std::vector<std::pair<int, int>>> partition_blocks(int tiles, int nk, const std::vector<double>& w) {
  const int n_sms = (int)w.size();
  const long long total = (long long)tiles * nk;
  std::vector<std::vector<std::pair<int, int>>> out(n_sms);
  std::vector<double> cum(n_sms + 1, 0.0);
  for (int s = 0; s < n_sms; ++s) cum[s + 1] = cum[s] + w[s];
  auto bound = [&](int s) { return (long long)std::llround(total * (cum[s] / cum[n_sms])); };
  for (int s = 0; s < n_sms; ++s) {
    long long a = bound(s);
    const long long b = bound(s + 1);
    while (a < b) {
      const long long tile_end = (a / nk + 1) * nk;
      const long long e = std::min(std::min(b, tile_end), a + kTcUnitsMax);
      out[s].push_back({(int)a, (int)(e - a)});
      a = e;
    }
  }
  return out;
}

Task make_task(uint8_t kind, int layer, int row0, int nrows) {
  Task t;
  std::memset(&t, 0, sizeof(t));
  t.kind = kind;
  t.layer = (uint16_t)layer;
  t.row0 = (uint32_t)row0;
  t.nrows = (uint32_t)nrows;
  return t;
}

bool is_gemv_kind(int k) {
  return k == TK_QKV || k == TK_OPROJ || k == TK_GATEUP || k == TK_DOWN || k == TK_LMHEAD;
}

void add_wait(Task& t, int e) { t.wait[t.n_wait++] = (uint32_t)e; }
void add_notify(Task& t, int e) { t.notify[t.n_notify++] = (uint32_t)e; }

// ---------------------------------------------------------------------------------------
// Validation of a task graph (used at build time and by mk_validate_taskgraph).
struct VTask {
  int kind, layer, sm, row0, nrows, n_wait, wait[2], n_notify, notify[2];
};

int validate(mk_ctx* c, const std::vector<VTask>& T, const std::vector<uint32_t>& cnt) {
  const mk_config& f = c->cfg;
  const int L = f.n_layers, nkv = f.n_kv_heads, nE = (int)cnt.size();
  const int rpg = c->rows_qkv / nkv;
  const int B = f.max_batch;
  char buf[256];
  // (a) ids
  for (size_t i = 0; i < T.size(); ++i) {
    const VTask& t = T[i];
    if (t.sm < 0 || t.sm >= c->n_sms || t.n_wait < 0 || t.n_wait > 2 || t.n_notify < 0 || t.n_notify > 2 ||
        t.layer < 0 || t.layer > L)
      return fail(c, MK_ERR_INVALID_ARG, "task " + std::to_string(i) + ": field out of range");
    for (int k = 0; k < t.n_wait; ++k)
      if (t.wait[k] < 0 || t.wait[k] >= nE) return fail(c, MK_ERR_INVALID_ARG, "task wait event out of range");
    for (int k = 0; k < t.n_notify; ++k)
      if (t.notify[k] < 0 || t.notify[k] >= nE)
        return fail(c, MK_ERR_INVALID_ARG, "task notify event out of range");
  }
  // (b) thresholds equal producer counts (every attention chunk task counts once per step,
  // whether its group's merge adds the counts of all its chunks or each head task its own)
  std::vector<uint32_t> produced(nE, 0);
  {
    for (const VTask& t : T)
      for (int k = 0; k < t.n_notify; ++k) produced[t.notify[k]]++;
    if (c->tc) {  // the last task of each LM tile counts
      std::vector<char> seen((size_t)c->tc_tiles[TK_LMHEAD], 0);
      for (const VTask& t : T)
        if (t.kind == TK_LMHEAD && t.row0 >= 0 && t.row0 / c->tc_nk[TK_LMHEAD] < c->tc_tiles[TK_LMHEAD] &&
            !seen[t.row0 / c->tc_nk[TK_LMHEAD]]) {
          seen[t.row0 / c->tc_nk[TK_LMHEAD]] = 1;
          produced[c->ev_lm]++;
        }
    } else {
      for (const VTask& t : T)
        if (t.kind == TK_LMHEAD) produced[c->ev_lm]++;
    }
    if (c->ev_tok < nE) produced[c->ev_tok] = 1;  // raised once per step by the token pick
  }
  for (int e = 0; e < nE; ++e)
    if (produced[e] != cnt[e]) {
      snprintf(buf, sizeof buf, "event %d: threshold %u but %u producers per step", e, cnt[e], produced[e]);
      return fail(c, MK_ERR_INVALID_ARG, buf);
    }
  // (c) every op's rows covered exactly once
  auto rows_of = [&](int kind) -> int {
    if (c->tc && kind != TK_EMBED) return c->tc_tiles[kind] * c->tc_nk[kind];  // weight blocks
    switch (kind) {
      case TK_EMBED: return f.hidden;
      case TK_QKV: return c->rows_qkv;
      case TK_OPROJ: return f.hidden;
      case TK_GATEUP: return c->rows_gu;
      case TK_DOWN: return f.hidden;
      case TK_LMHEAD: return f.vocab;
    }
    return 0;
  };
  std::vector<std::vector<int>> cover((size_t)8 * (L + 1));
  std::vector<std::vector<int>> attn_cover((size_t)L * B * nkv);
  for (const VTask& t : T) {
    if (t.kind == TK_ATTN) {
      if (t.row0 < 0 || t.row0 >= B * nkv || t.layer >= L)
        return fail(c, MK_ERR_INVALID_ARG, "attention task outside the (sequence, KV head) range");
      auto& v = attn_cover[(size_t)t.layer * B * nkv + t.row0];
      v.push_back(t.nrows);  // chunk index travels in nrows of the export
      continue;
    }
    if (t.kind < TK_EMBED || t.kind > TK_LMHEAD) return fail(c, MK_ERR_INVALID_ARG, "unknown task kind");
    int rows = rows_of(t.kind);
    if (t.nrows <= 0 || t.nrows > c->task_rows || t.row0 < 0 || t.row0 + t.nrows > rows)
      return fail(c, MK_ERR_INVALID_ARG, "task rows out of range");
    if (c->tc && t.kind != TK_EMBED && t.row0 / c->tc_nk[t.kind] != (t.row0 + t.nrows - 1) / c->tc_nk[t.kind])
      return fail(c, MK_ERR_INVALID_ARG, "a tensor-core task spans two tiles");
    if (!c->tc && (t.kind == TK_QKV || t.kind == TK_GATEUP) && ((t.row0 | t.nrows) & 1))
      return fail(c, MK_ERR_INVALID_ARG, "QKV/gate-up tasks must hold whole row pairs");
    int lay = (t.kind == TK_EMBED || t.kind == TK_LMHEAD) ? L : t.layer;
    auto& v = cover[(size_t)t.kind * (L + 1) + lay];
    if (v.empty()) v.assign(rows, 0);
    for (int r = t.row0; r < t.row0 + t.nrows; ++r) v[r]++;
  }
  for (int kind = TK_EMBED; kind <= TK_LMHEAD; ++kind) {
    if (kind == TK_ATTN) continue;
    for (int l = 0; l <= L; ++l) {
      bool per_layer = !(kind == TK_EMBED || kind == TK_LMHEAD);
      if (per_layer == (l == L)) continue;
      auto& v = cover[(size_t)kind * (L + 1) + l];
      int rows = rows_of(kind);
      if ((int)v.size() != rows) return fail(c, MK_ERR_INVALID_ARG, "an op has no tasks");
      const int want = (kind == TK_DOWN) ? c->ndc : 1;  // one down task per K chunk
      for (int r = 0; r < rows; ++r)
        if (v[r] != want) {
          snprintf(buf, sizeof buf, "op kind %d layer %d: row %d covered %d times", kind, l, r, v[r]);
          return fail(c, MK_ERR_INVALID_ARG, buf);
        }
    }
  }
  for (int l = 0; l < L; ++l)
    for (int bg = 0; bg < B * nkv; ++bg) {
      auto v = attn_cover[(size_t)l * B * nkv + bg];
      std::sort(v.begin(), v.end());
      bool ok = (int)v.size() == c->nch;
      for (int i = 0; ok && i < (int)v.size(); ++i) ok = v[i] == i;
      if (!ok) return fail(c, MK_ERR_INVALID_ARG, "attention chunks of a (sequence, KV head) incomplete");
    }
  // (d) simulate the queues: deadlock-freedom; (e) every read after its writes
  // categories: 0 embed; per layer: qkv-group g, qkv, attn, o, gu, down; last: lm
  const int CPL = nkv + 5;
  auto cat_qkvg = [&](int l, int g) { return 1 + l * CPL + g; };
  auto cat_of = [&](int kind, int l) {
    switch (kind) {
      case TK_QKV: return 1 + l * CPL + nkv;
      case TK_ATTN: return 1 + l * CPL + nkv + 1;
      case TK_OPROJ: return 1 + l * CPL + nkv + 2;
      case TK_GATEUP: return 1 + l * CPL + nkv + 3;
      case TK_DOWN: return 1 + l * CPL + nkv + 4;
      case TK_LMHEAD: return 1 + L * CPL;
    }
    return 0;
  };
  const int NC = 2 + L * CPL;
  const int W = (NC + 63) / 64;
  std::vector<int> cat_size(NC, 0);
  auto cats_of_task = [&](const VTask& t, std::vector<int>& out) {
    out.clear();
    out.push_back(cat_of(t.kind, t.layer));
    if (t.kind == TK_QKV) {
      int r0 = t.row0, r1 = t.row0 + t.nrows - 1;  // packed rows written (by the tile, for tensor-core tasks)
      if (c->tc) {
        const int tile = t.row0 / c->tc_nk[TK_QKV];
        r0 = tile * kTcRows;
        r1 = std::min(c->rows_qkv, r0 + kTcRows) - 1;
      }
      for (int g = r0 / rpg; g <= r1 / rpg; ++g) out.push_back(cat_qkvg(t.layer, g));
    }
  };
  std::vector<int> tmp;
  for (const VTask& t : T) {
    cats_of_task(t, tmp);
    for (int x : tmp) cat_size[x]++;
  }
  // per-SM queues in array order
  std::vector<std::vector<int>> q(c->n_sms);
  for (size_t i = 0; i < T.size(); ++i) q[T[i].sm].push_back((int)i);
  std::vector<size_t> head(c->n_sms, 0);
  std::vector<uint32_t> ctr(nE, 0);
  std::vector<uint64_t> Gb(T.size() * W, 0);   // categories complete before the task starts
  std::vector<uint64_t> Fe((size_t)nE * W, 0);  // categories complete when the event is active
  std::vector<std::vector<int>> ev_cat_done(nE, std::vector<int>());
  std::vector<int> cat_done(NC, 0);
  std::vector<int> attn_arrive((size_t)L * B * nkv, 0);
  std::vector<uint64_t> attn_acc((size_t)L * B * nkv * W, 0);
  auto setbit = [&](uint64_t* bs, int x) { bs[x >> 6] |= 1ull << (x & 63); };
  auto hasbit = [&](const uint64_t* bs, int x) { return (bs[x >> 6] >> (x & 63)) & 1ull; };
  std::vector<int> ev_ncat((size_t)nE * NC, 0);  // notifiers of e per category (for "all of C done")
  size_t executed = 0;
  std::vector<uint64_t> prevG(W);
  std::vector<std::vector<uint64_t>> smG(c->n_sms, std::vector<uint64_t>(W, 0));
  auto fire = [&](int e, const uint64_t* contrib, const std::vector<int>& cats_done) {
    ctr[e]++;
    for (int w = 0; w < W; ++w) Fe[(size_t)e * W + w] |= contrib[w];
    for (int x : cats_done) {
      int& n = ev_ncat[(size_t)e * NC + x];
      n++;
      if (n == cat_size[x]) setbit(&Fe[(size_t)e * W], x);
    }
  };
  bool progress = true;
  while (progress) {
    progress = false;
    for (int s = 0; s < c->n_sms; ++s) {
      while (head[s] < q[s].size()) {
        const int i = q[s][head[s]];
        const VTask& t = T[i];
        bool ready = true;
        for (int k = 0; k < t.n_wait; ++k)
          if (ctr[t.wait[k]] < cnt[t.wait[k]]) ready = false;
        if (!ready) break;
        // categories complete before t: its queue predecessor's view plus the waited events'
        uint64_t* gi = &Gb[(size_t)i * W];
        for (int w = 0; w < W; ++w) gi[w] = smG[s][w];
        for (int k = 0; k < t.n_wait; ++k)
          for (int w = 0; w < W; ++w) gi[w] |= Fe[(size_t)t.wait[k] * W + w];
        // required inputs
        std::vector<int> need;
        const int l = t.layer;
        switch (t.kind) {
          case TK_QKV: need.push_back(l == 0 ? 0 : cat_of(TK_DOWN, l - 1)); break;
          case TK_ATTN: need.push_back(cat_qkvg(l, t.row0 % nkv)); break;
          case TK_OPROJ:
            need.push_back(cat_of(TK_ATTN, l));
            need.push_back(l == 0 ? 0 : cat_of(TK_DOWN, l - 1));
            break;
          case TK_GATEUP: need.push_back(cat_of(TK_OPROJ, l)); break;
          case TK_DOWN:
            need.push_back(cat_of(TK_GATEUP, l));
            need.push_back(cat_of(TK_OPROJ, l));
            break;
          case TK_LMHEAD: need.push_back(cat_of(TK_DOWN, L - 1)); break;
        }
        for (int x : need)
          if (!hasbit(gi, x)) {
            snprintf(buf, sizeof buf, "task %d (kind %d layer %d) may read data before its producers finish", i,
                     t.kind, l);
            return fail(c, MK_ERR_INVALID_ARG, buf);
          }
        // execute
        cats_of_task(t, tmp);
        for (int x : tmp) {
          if (++cat_done[x] == cat_size[x]) { /* completion is only visible through events */ }
        }
        if (t.kind == TK_ATTN) {
          size_t key = (size_t)l * B * nkv + t.row0;
          uint64_t* acc = &attn_acc[key * W];
          for (int w = 0; w < W; ++w) acc[w] |= gi[w];
          if (++attn_arrive[key] == c->nch) {
            // the merge runs after every chunk of the group: all their views hold, and the
            // group's chunks are done; it adds one count per chunk (head mode adds the same
            // counts from the chunks themselves, the last of them after every head's output)
            std::vector<int> done_cats, none;
            for (int r = 0; r < c->nch; ++r) done_cats.push_back(cat_of(TK_ATTN, l));
            for (int k = 0; k < t.n_notify; ++k)
              for (int r = 0; r < c->nch; ++r) fire(t.notify[k], acc, r == 0 ? done_cats : none);
          }
        } else {
          for (int k = 0; k < t.n_notify; ++k) fire(t.notify[k], gi, tmp);
        }
        if (t.kind == TK_LMHEAD) ctr[c->ev_lm]++;
        head[s]++;
        executed++;
        progress = true;
      }
    }
  }
  if (executed != T.size()) {
    for (int s = 0; s < c->n_sms; ++s)
      if (head[s] < q[s].size()) {
        snprintf(buf, sizeof buf, "deadlock: SM %d blocked at its task %zu (graph task %d)", s, head[s],
                 q[s][head[s]]);
        return fail(c, MK_ERR_INVALID_ARG, buf);
      }
  }
  return MK_OK;
}

std::vector<VTask> to_vtasks(const Graph& g) {
  std::vector<VTask> v;
  for (const TaskRec& r : g.tasks) {
    VTask t;
    t.kind = r.t.kind;
    t.layer = r.t.layer;
    t.sm = r.sm;
    t.row0 = (int)r.t.row0;
    t.nrows = r.t.kind == TK_ATTN ? (int)r.t.aux : (int)r.t.nrows;
    t.n_wait = r.t.n_wait;
    t.wait[0] = (int)r.t.wait[0];
    t.wait[1] = (int)r.t.wait[1];
    t.n_notify = r.t.n_notify;
    t.notify[0] = (int)r.t.notify[0];
    t.notify[1] = (int)r.t.notify[1];
    v.push_back(t);
  }
  return v;
}

// ---------------------------------------------------------------------------------------
// Validation of a tensor-parallel graph (every rank's tasks; used when an emulated
// tensor-parallel context is built and by mk_validate_taskgraph_tp).  A task's events live on
// its own rank; a remote-signal edge (remote = 1) raises the notified event on every rank.
// Checks, per rank: thresholds equal the producers that reach the rank's counter; every op's
// rows and every attention chunk covered once; the summed residual rows written once per
// layer (gate/up writes x_mid); and, simulating every rank's
// queues together, no deadlock and no task reading data before its producers -- on its own
// rank or, for the receive buffers of the row-parallel projections, on every rank.
struct TVTask {
  int rank, kind, layer, sm, row0, nrows, n_wait, wait[2], n_notify, notify[2], remote, mlo, mhi;
};

int validate_tp(mk_ctx* c, const std::vector<TVTask>& T, const std::vector<uint32_t>& cnt) {
  const mk_ctx* sh = c->tp_shards[0];
  const mk_config& f = sh->cfg;  // one rank's shapes
  const int R = c->tp_ranks, S = c->tp_sms, L = f.n_layers, nkv = f.n_kv_heads, B = f.max_batch, H = f.hidden;
  const int nE = (int)cnt.size();
  const int rpg = sh->rows_qkv / nkv;
  char buf[256];
  if (nE != sh->n_events) return fail(c, MK_ERR_INVALID_ARG, "event count array has the wrong length");
  for (size_t i = 0; i < T.size(); ++i) {
    const TVTask& t = T[i];
    if (t.rank < 0 || t.rank >= R || t.sm < t.rank * S || t.sm >= (t.rank + 1) * S || t.n_wait < 0 || t.n_wait > 2 ||
        t.n_notify < 0 || t.n_notify > 2 || t.layer < 0 || t.layer > L || (t.remote != 0 && t.remote != 1))
      return fail(c, MK_ERR_INVALID_ARG, "task " + std::to_string(i) + ": field out of range");
    for (int k = 0; k < t.n_wait; ++k)
      if (t.wait[k] < 0 || t.wait[k] >= nE) return fail(c, MK_ERR_INVALID_ARG, "task wait event out of range");
    for (int k = 0; k < t.n_notify; ++k)
      if (t.notify[k] < 0 || t.notify[k] >= nE) return fail(c, MK_ERR_INVALID_ARG, "task notify event out of range");
  }
  // (b) thresholds, per rank
  std::vector<uint32_t> produced((size_t)R * nE, 0);
  {
    for (const TVTask& t : T) {
      for (int k = 0; k < t.n_notify; ++k) {
        // every attention chunk task counts once per step (see the single-device check)
        for (int d = 0; d < R; ++d)
          if (t.remote || d == t.rank) produced[(size_t)d * nE + t.notify[k]]++;
      }
      if (t.kind == TK_LMHEAD) produced[(size_t)t.rank * nE + sh->ev_lm]++;
    }
    for (int r = 0; r < R; ++r) {
      produced[(size_t)r * nE + sh->ev_tok] = 1;                    // the rank's token pick
      produced[(size_t)r * nE + sh->ev_lmx] = (uint32_t)(R * B);  // every rank's argmax exchange
    }
  }
  for (int r = 0; r < R; ++r)
    for (int e = 0; e < nE; ++e)
      if (produced[(size_t)r * nE + e] != cnt[e]) {
        snprintf(buf, sizeof buf, "rank %d event %d: threshold %u but %u producers per step", r, e, cnt[e],
                 produced[(size_t)r * nE + e]);
        return fail(c, MK_ERR_INVALID_ARG, buf);
      }
  // (c) coverage per rank: op rows, attention chunks, materialised residual rows
  auto rows_of = [&](int kind) -> int {
    switch (kind) {
      case TK_EMBED: return H;
      case TK_QKV: return sh->rows_qkv;
      case TK_OPROJ: return H;
      case TK_GATEUP: return sh->rows_gu;
      case TK_DOWN: return H;
      case TK_LMHEAD: return f.vocab;
    }
    return 0;
  };
  for (int r = 0; r < R; ++r) {
    std::vector<std::vector<int>> cover((size_t)8 * (L + 1)), mat((size_t)L);
    std::vector<std::vector<int>> attn_cover((size_t)L * B * nkv);
    for (const TVTask& t : T) {
      if (t.rank != r) continue;
      if (t.kind == TK_ATTN) {
        if (t.row0 < 0 || t.row0 >= B * nkv || t.layer >= L)
          return fail(c, MK_ERR_INVALID_ARG, "attention task outside the (sequence, KV head) range");
        attn_cover[(size_t)t.layer * B * nkv + t.row0].push_back(t.nrows);
        continue;
      }
      if (t.kind < TK_EMBED || t.kind > TK_LMHEAD) return fail(c, MK_ERR_INVALID_ARG, "unknown task kind");
      const int rows = rows_of(t.kind);
      if (t.nrows <= 0 || t.nrows > sh->task_rows || t.row0 < 0 || t.row0 + t.nrows > rows)
        return fail(c, MK_ERR_INVALID_ARG, "task rows out of range");
      if ((t.kind == TK_QKV || t.kind == TK_GATEUP) && ((t.row0 | t.nrows) & 1))
        return fail(c, MK_ERR_INVALID_ARG, "QKV/gate-up tasks must hold whole row pairs");
      const int lay = (t.kind == TK_EMBED || t.kind == TK_LMHEAD) ? L : t.layer;
      auto& v = cover[(size_t)t.kind * (L + 1) + lay];
      if (v.empty()) v.assign(rows, 0);
      for (int x = t.row0; x < t.row0 + t.nrows; ++x) v[x]++;
      if (t.kind == TK_GATEUP) {
        if (t.mlo < 0 || t.mhi < t.mlo || t.mhi > H || ((t.mlo | t.mhi) & 7))
          return fail(c, MK_ERR_INVALID_ARG, "residual slice out of range or not a multiple of 8");
        auto& m = mat[t.layer];
        if (m.empty()) m.assign(H, 0);
        for (int x = t.mlo; x < t.mhi; ++x) m[x]++;
      }
    }
    for (int kind = TK_EMBED; kind <= TK_LMHEAD; ++kind) {
      if (kind == TK_ATTN) continue;
      for (int l = 0; l <= L; ++l) {
        const bool per_layer = !(kind == TK_EMBED || kind == TK_LMHEAD);
        if (per_layer == (l == L)) continue;
        auto& v = cover[(size_t)kind * (L + 1) + l];
        if ((int)v.size() != rows_of(kind)) return fail(c, MK_ERR_INVALID_ARG, "an op has no tasks on a rank");
        for (int x = 0; x < (int)v.size(); ++x)
          if (v[x] != 1) {
            snprintf(buf, sizeof buf, "rank %d op kind %d layer %d: row %d covered %d times", r, kind, l, x, v[x]);
            return fail(c, MK_ERR_INVALID_ARG, buf);
          }
      }
    }
    for (int l = 0; l < L; ++l) {
      const auto& m = mat[l];
      for (int x = 0; x < H; ++x)
        if ((m.empty() ? 0 : m[x]) != 1) {
          snprintf(buf, sizeof buf, "rank %d layer %d: residual row %d of x_mid written %d times", r, l, x,
                   m.empty() ? 0 : m[x]);
          return fail(c, MK_ERR_INVALID_ARG, buf);
        }
    }
    for (int l = 0; l < L; ++l)
      for (int bg = 0; bg < B * nkv; ++bg) {
        auto v = attn_cover[(size_t)l * B * nkv + bg];
        std::sort(v.begin(), v.end());
        bool ok = (int)v.size() == sh->nch;
        for (int i = 0; ok && i < (int)v.size(); ++i) ok = v[i] == i;
        if (!ok) return fail(c, MK_ERR_INVALID_ARG, "attention chunks of a (sequence, KV head) incomplete");
      }
  }
  // (d) + (e): every rank's queues together; categories and events per rank
  const int CPL = nkv + 5, NC = 2 + L * CPL, NCA = R * NC, W = (NCA + 63) / 64;
  auto cat_qkvg = [&](int r, int l, int g) { return r * NC + 1 + l * CPL + g; };
  auto cat_of = [&](int r, int kind, int l) {
    switch (kind) {
      case TK_QKV: return r * NC + 1 + l * CPL + nkv;
      case TK_ATTN: return r * NC + 1 + l * CPL + nkv + 1;
      case TK_OPROJ: return r * NC + 1 + l * CPL + nkv + 2;
      case TK_GATEUP: return r * NC + 1 + l * CPL + nkv + 3;
      case TK_DOWN: return r * NC + 1 + l * CPL + nkv + 4;
      case TK_LMHEAD: return r * NC + 1 + L * CPL;
    }
    return r * NC;  // embedding
  };
  std::vector<int> cat_size(NCA, 0), tmp;
  auto cats_of_task = [&](const TVTask& t, std::vector<int>& out) {
    out.clear();
    out.push_back(cat_of(t.rank, t.kind, t.layer));
    if (t.kind == TK_QKV)
      for (int g = t.row0 / rpg; g <= (t.row0 + t.nrows - 1) / rpg; ++g) out.push_back(cat_qkvg(t.rank, t.layer, g));
  };
  for (const TVTask& t : T) {
    cats_of_task(t, tmp);
    for (int x : tmp) cat_size[x]++;
  }
  const int NS = R * S;
  std::vector<std::vector<int>> q(NS);
  for (size_t i = 0; i < T.size(); ++i) q[T[i].sm].push_back((int)i);
  std::vector<size_t> head(NS, 0);
  std::vector<uint32_t> ctr((size_t)R * nE, 0);
  std::vector<uint64_t> Gb(W, 0), Fe((size_t)R * nE * W, 0);
  std::vector<int> ev_ncat((size_t)R * nE * NCA, 0);
  std::vector<int> attn_arrive((size_t)R * L * B * nkv, 0);
  std::vector<uint64_t> attn_acc((size_t)R * L * B * nkv * W, 0);
  std::vector<std::vector<uint64_t>> smG(NS, std::vector<uint64_t>(W, 0));
  auto setbit = [&](uint64_t* bs, int x) { bs[x >> 6] |= 1ull << (x & 63); };
  auto hasbit = [&](const uint64_t* bs, int x) { return (bs[x >> 6] >> (x & 63)) & 1ull; };
  auto fire = [&](int r, int e, const uint64_t* contrib, const std::vector<int>& cats_done) {
    const size_t ge = (size_t)r * nE + e;
    ctr[ge]++;
    for (int w = 0; w < W; ++w) Fe[ge * W + w] |= contrib[w];
    for (int x : cats_done)
      if (++ev_ncat[ge * NCA + x] == cat_size[x]) setbit(&Fe[ge * W], x);
  };
  size_t executed = 0;
  bool progress = true;
  while (progress) {
    progress = false;
    for (int sm = 0; sm < NS; ++sm) {
      while (head[sm] < q[sm].size()) {
        const int i = q[sm][head[sm]];
        const TVTask& t = T[i];
        const int r = t.rank, l = t.layer;
        bool ready = true;
        for (int k = 0; k < t.n_wait; ++k)
          if (ctr[(size_t)r * nE + t.wait[k]] < cnt[t.wait[k]]) ready = false;
        if (!ready) break;
        for (int w = 0; w < W; ++w) Gb[w] = smG[sm][w];
        for (int k = 0; k < t.n_wait; ++k)
          for (int w = 0; w < W; ++w) Gb[w] |= Fe[((size_t)r * nE + t.wait[k]) * W + w];
        std::vector<int> need;
        auto all_ranks = [&](int kind, int layer) {
          for (int d = 0; d < R; ++d) need.push_back(cat_of(d, kind, layer));
        };
        switch (t.kind) {
          case TK_QKV:
            if (l == 0) {
              need.push_back(cat_of(r, TK_EMBED, 0));
            } else {
              all_ranks(TK_DOWN, l - 1);                    // the ranks' down rows
              need.push_back(cat_of(r, TK_GATEUP, l - 1));  // x_mid[l-1], materialised by this rank
            }
            break;
          case TK_ATTN: need.push_back(cat_qkvg(r, l, t.row0 % nkv)); break;
          case TK_OPROJ: need.push_back(cat_of(r, TK_ATTN, l)); break;
          case TK_GATEUP:
            all_ranks(TK_OPROJ, l);  // the ranks' O rows
            if (l == 0) {
              need.push_back(cat_of(r, TK_EMBED, 0));
            } else {                                        // x_in[l], formed as in QKV
              all_ranks(TK_DOWN, l - 1);
              need.push_back(cat_of(r, TK_GATEUP, l - 1));
            }
            break;
          case TK_DOWN: need.push_back(cat_of(r, TK_GATEUP, l)); break;
          case TK_LMHEAD:
            all_ranks(TK_DOWN, L - 1);
            need.push_back(cat_of(r, TK_GATEUP, L - 1));
            break;
        }
        for (int x : need)
          if (!hasbit(Gb.data(), x)) {
            snprintf(buf, sizeof buf, "rank %d task %d (kind %d layer %d) may read data before its producers finish",
                     r, i, t.kind, l);
            return fail(c, MK_ERR_INVALID_ARG, buf);
          }
        cats_of_task(t, tmp);
        if (t.kind == TK_ATTN) {
          const size_t key = ((size_t)r * L + l) * B * nkv + t.row0;
          uint64_t* acc = &attn_acc[key * W];
          for (int w = 0; w < W; ++w) acc[w] |= Gb[w];
          if (++attn_arrive[key] == sh->nch) {
            std::vector<int> done(sh->nch, cat_of(r, TK_ATTN, l)), none;
            for (int k = 0; k < t.n_notify; ++k)
              for (int d = 0; d < R; ++d)
                if (t.remote || d == r)
                  for (int x = 0; x < sh->nch; ++x) fire(d, t.notify[k], acc, x == 0 ? done : none);
          }
        } else {
          for (int k = 0; k < t.n_notify; ++k)
            for (int d = 0; d < R; ++d)
              if (t.remote || d == r) fire(d, t.notify[k], Gb.data(), tmp);
        }
        for (int w = 0; w < W; ++w) smG[sm][w] = Gb[w];
        head[sm]++;
        executed++;
        progress = true;
      }
    }
  }
  if (executed != T.size()) {
    for (int sm = 0; sm < NS; ++sm)
      if (head[sm] < q[sm].size()) {
        snprintf(buf, sizeof buf, "deadlock: SM %d (rank %d) blocked at its task %zu", sm, sm / S, head[sm]);
        return fail(c, MK_ERR_INVALID_ARG, buf);
      }
  }
  return MK_OK;
}

std::vector<TVTask> tp_vtasks(const mk_ctx* c) {
  std::vector<TVTask> v;
  for (size_t i = 0; i < c->tp_tasks.size(); ++i) {
    const Task& t = c->tp_tasks[i];
    const int sm = c->tp_task_sm[i];
    TVTask x;
    x.rank = sm / c->tp_sms;
    x.kind = t.kind;
    x.layer = t.layer;
    x.sm = sm;
    x.row0 = (int)t.row0;
    x.nrows = t.kind == TK_ATTN ? (int)t.aux : (int)t.nrows;
    x.n_wait = t.n_wait;
    x.wait[0] = (int)t.wait[0];
    x.wait[1] = (int)t.wait[1];
    x.n_notify = t.n_notify;
    x.notify[0] = (int)t.notify[0];
    x.notify[1] = (int)t.notify[1];
    x.remote = (t.kind == TK_OPROJ || t.kind == TK_DOWN) ? (t.pad0 & 1) : 0;
    x.mlo = t.kind == TK_GATEUP ? (int)t.index : 0;
    x.mhi = t.kind == TK_GATEUP ? (int)t.pad1 : 0;
    v.push_back(x);
  }
  return v;
}

// Tensor parallel: the tasks of op `kind` in layer l (queue order, SM 0 first) share out the
// rows [0, H) of the residual sum they form, each writing its slice [index, pad1) (multiples
// of 8, so whole 8-element groups of a GEMV thread's input).
void share_rows(std::vector<std::vector<Task>>& q, int kind, int l, int H) {
  std::vector<Task*> ts;
  for (auto& v : q)
    for (auto& t : v)
      if (t.kind == kind && t.layer == l) ts.push_back(&t);
  const int n = (int)ts.size();
  for (int j = 0; j < n; ++j) {
    ts[j]->index = (uint32_t)((long long)H * j / n / 8 * 8);
    ts[j]->pad1 = (uint32_t)(j + 1 == n ? H : (long long)H * (j + 1) / n / 8 * 8);
  }
}

// ---------------------------------------------------------------------------------------
int build_graph(mk_ctx* c) {
  const mk_config& f = c->cfg;
  const int L = f.n_layers, nkv = f.n_kv_heads, D = f.head_dim, n = c->n_sms;
  const int B = f.max_batch;
  const bool tp = c->tp_ranks > 1;
  c->n_events = 1 + L * (nkv + 4) + 2 + (tp ? 1 : 0);
  c->ev_lm = 1 + L * (nkv + 4);
  c->ev_tok = c->ev_lm + 1;  // tokens picked: a later step of a multi-step launch waits on it
  c->ev_lmx = tp ? c->ev_lm + 2 : -1;  // tensor parallel: every rank's argmax partial arrived
  std::vector<uint32_t> evc(c->n_events, 0);
  std::vector<std::vector<Task>> q(n);
  const int rpg = (c->G + 2) * D;
  // Run-time claims (mk_set_dispatch): a projection of a layer is a pool of tasks cut for
  // n_sms * dyn_split equal shares; every SM's queue holds one TK_POOL entry for it, where the
  // SM claims tasks until the pool is empty.  qv is the validation view: the pool's tasks
  // dealt round-robin over the SMs at that queue position (one assignment the claims can give).
  const bool dyn = c->dyn != 0;
  std::vector<std::vector<Task>> qv(n);

  // embedding slices
  {
    auto parts = partition_rows(f.hidden, 1, c->sm_weights, c->task_rows);
    for (int s = 0; s < n; ++s)
      for (auto& p : parts[s]) {
        Task t = make_task(TK_EMBED, 0, p.first, p.second);
        add_notify(t, ev_embed());
        evc[ev_embed()]++;
        q[s].push_back(t);
        if (dyn) qv[s].push_back(t);
      }
  }
  // GEMV ops.  CUDA-core tasks: row ranges (parts = (first row, rows)).  Tensor-core tasks:
  // block ranges of one tile (parts = (first block, blocks)); the tile's tasks get slots in
  // SM order, and its partial records are rec0[tile] + slot (the same for every layer).
  struct Plan {
    std::vector<std::vector<std::pair<int, int>>> parts;
    std::vector<std::vector<int>> slot;  // tensor-core: per SM, per part
    std::vector<int> nsplit, rec0;       // tensor-core: per tile
  };
  size_t rec_next = 0;
  auto op_w = [&](int kind) -> const std::vector<double>& {
    return c->op_weights[kind].empty() ? c->sm_weights : c->op_weights[kind];
  };
  auto plan = [&](int kind, int rows, int gran) {
    Plan pl;
    if (!c->tc) {
      pl.parts = partition_rows(rows, gran, op_w(kind), c->task_rows);
      return pl;
    }
    const int nk = c->tc_nk[kind], tiles = c->tc_tiles[kind];
    pl.parts = partition_blocks(tiles, nk, op_w(kind));
    pl.nsplit.assign(tiles, 0);
    pl.slot.resize(n);
    for (int s = 0; s < n; ++s)
      for (auto& p : pl.parts[s]) pl.slot[s].push_back(pl.nsplit[p.first / nk]++);
    pl.rec0.assign(tiles, 0);
    for (int t = 0; t < tiles; ++t) {
      pl.rec0[t] = (int)rec_next;
      rec_next += pl.nsplit[t];
    }
    return pl;
  };
  auto gemv_task = [&](int kind, int l, const Plan& pl, int s, int j) {
    const auto& p = pl.parts[s][j];
    Task t = make_task(kind, l, p.first, p.second);
    if (c->tc) {
      const int tile = p.first / c->tc_nk[kind];
      t.aux = (uint16_t)pl.slot[s][j];
      t.pad0 = (uint8_t)pl.nsplit[tile];
      t.index = (uint32_t)(pl.rec0[tile] + pl.slot[s][j]);
      t.pad1 = (uint32_t)((kind == TK_LMHEAD ? 0 : l) * c->n_tile_ids + c->tc_tile_base[kind] + tile);
    }
    return t;
  };
  if (c->tc)
    for (int k : {TK_QKV, TK_OPROJ, TK_GATEUP, TK_DOWN, TK_LMHEAD})
      if (c->tc_tiles[k] * c->tc_nk[k] > 0 && c->tc_nk[k] > 255)
        return fail(c, MK_ERR_UNSUPPORTED, "K too large for the tensor-core tile split");
  const Plan qkv_pl = plan(TK_QKV, c->rows_qkv, 2);
  const Plan o_pl = plan(TK_OPROJ, f.hidden, 1);
  const Plan gu_pl = plan(TK_GATEUP, c->rows_gu, 2);
  const Plan d_pl = plan(TK_DOWN, f.hidden, 1);
  const Plan lm_pl = plan(TK_LMHEAD, f.vocab, 1);
  c->n_recs = rec_next;
  const int n_attn = B * nkv * c->nch;
  std::vector<Task> pool_tasks;
  c->pool_first.clear();
  c->pool_count.clear();
  auto push_static = [&](int s, const Task& t) {
    q[s].push_back(t);
    if (dyn) qv[s].push_back(t);
  };
  auto add_pool = [&](int kind, int l, int rows, int gran, auto&& finish) -> int {
    const auto parts = partition_rows(rows, gran, std::vector<double>((size_t)n * c->dyn_split, 1.0), c->task_rows);
    const uint32_t p = (uint32_t)c->pool_first.size();
    c->pool_first.push_back((uint32_t)pool_tasks.size());
    uint32_t cnt = 0;
    for (const auto& v : parts)
      for (const auto& pr : v) {
        Task t = make_task(kind, l, pr.first, pr.second);
        if (int rc = finish(t)) return rc;
        pool_tasks.push_back(t);
        qv[cnt % n].push_back(t);
        ++cnt;
      }
    c->pool_count.push_back(cnt);
    Task e = make_task(TK_POOL, l, 0, 0);
    e.index = p;
    for (int s2 = 0; s2 < n; ++s2) q[s2].push_back(e);
    return MK_OK;
  };
  for (int l = 0; l < L; ++l) {
    auto qkv_edges = [&](Task& t) -> int {
      add_wait(t, l == 0 ? ev_embed() : ev_down(c, l - 1));
      const int g0 = (int)t.row0 / rpg, g1 = (int)(t.row0 + t.nrows - 1) / rpg;
      if (g1 - g0 > 1) return fail(c, MK_ERR_UNSUPPORTED, "QKV task spans more than two KV groups");
      for (int g = g0; g <= g1; ++g) {
        add_notify(t, ev_qkv(c, l, g));
        evc[ev_qkv(c, l, g)]++;
      }
      return MK_OK;
    };
    if (dyn) {
      if (int rc = add_pool(TK_QKV, l, c->rows_qkv, 2, qkv_edges)) return rc;
    } else
    for (int s = 0; s < n; ++s)
      for (int j = 0; j < (int)qkv_pl.parts[s].size(); ++j) {
        Task t = gemv_task(TK_QKV, l, qkv_pl, s, j);
        add_wait(t, l == 0 ? ev_embed() : ev_down(c, l - 1));
        int r0 = (int)t.row0, r1 = (int)(t.row0 + t.nrows - 1);  // packed rows the task (or its tile) writes
        if (c->tc) {
          r0 = (int)t.row0 / c->tc_nk[TK_QKV] * kTcRows;
          r1 = std::min(c->rows_qkv, r0 + kTcRows) - 1;
        }
        const int g0 = r0 / rpg, g1 = r1 / rpg;
        if (g1 - g0 > 1) return fail(c, MK_ERR_UNSUPPORTED, "QKV tile spans more than two KV groups");
        for (int g = g0; g <= g1; ++g) {
          add_notify(t, ev_qkv(c, l, g));
          evc[ev_qkv(c, l, g)]++;
        }
        q[s].push_back(t);
      }
    // priority claims: the attention chunks (the critical path between QKV and O) become a pool
    // right after the QKV pool, taken by whichever SMs finish their QKV claims first
    const bool attn_pool = dyn && c->dyn == MK_DISPATCH_CLAIM_PRIORITY;
    const uint32_t attn_p = (uint32_t)c->pool_first.size();
    if (attn_pool) c->pool_first.push_back((uint32_t)pool_tasks.size());
    for (int idx = 0; idx < n_attn; ++idx) {
      const int bg = idx / c->nch, ch = idx % c->nch;
      const int g = bg % nkv;
      Task t = make_task(TK_ATTN, l, bg, 0);
      t.aux = (uint16_t)ch;
      add_wait(t, ev_qkv(c, l, g));
      add_notify(t, ev_attn(c, l));
      if (attn_pool) {
        pool_tasks.push_back(t);
        qv[idx % n].push_back(t);
        continue;
      }
      const int s = (int)(((long long)idx * n / n_attn + (long long)l * 37) % n);
      push_static(s, t);
    }
    if (attn_pool) {
      c->pool_count.push_back((uint32_t)n_attn);
      Task e = make_task(TK_POOL, l, 0, 0);
      e.index = attn_p;
      for (int s2 = 0; s2 < n; ++s2) q[s2].push_back(e);
    }
    // one count per chunk task and step: a split-mode merge adds its group's nch at once; in
    // head mode each head task adds its own and one chunk adds those of the chunks without work
    evc[ev_attn(c, l)] = (uint32_t)(B * nkv * c->nch);
    if (dyn) {
      auto o_edges = [&](Task& t) -> int {
        add_wait(t, ev_attn(c, l));
        add_notify(t, ev_o(c, l));
        evc[ev_o(c, l)]++;
        return MK_OK;
      };
      auto gu_edges = [&](Task& t) -> int {
        add_wait(t, ev_o(c, l));
        add_notify(t, ev_gu(c, l));
        evc[ev_gu(c, l)]++;
        return MK_OK;
      };
      auto d_edges = [&](Task& t) -> int {
        add_wait(t, ev_gu(c, l));
        add_notify(t, ev_down(c, l));
        evc[ev_down(c, l)]++;
        return MK_OK;
      };
      if (int rc = add_pool(TK_OPROJ, l, f.hidden, 1, o_edges)) return rc;
      if (int rc = add_pool(TK_GATEUP, l, c->rows_gu, 2, gu_edges)) return rc;
      if (int rc = add_pool(TK_DOWN, l, f.hidden, 1, d_edges)) return rc;
      continue;
    }
    for (int s = 0; s < n; ++s)
      for (int j = 0; j < (int)o_pl.parts[s].size(); ++j) {
        Task t = gemv_task(TK_OPROJ, l, o_pl, s, j);
        add_wait(t, ev_attn(c, l));
        add_notify(t, ev_o(c, l));
        if (tp) t.pad0 = 1;  // remote-signal edge: the partial rows go to every rank
        evc[ev_o(c, l)] += tp ? (uint32_t)c->tp_ranks : 1u;
        q[s].push_back(t);
      }
    for (int s = 0; s < n; ++s)
      for (int j = 0; j < (int)gu_pl.parts[s].size(); ++j) {
        Task t = gemv_task(TK_GATEUP, l, gu_pl, s, j);
        add_wait(t, ev_o(c, l));
        add_notify(t, ev_gu(c, l));
        evc[ev_gu(c, l)]++;
        q[s].push_back(t);
      }
    if (tp) share_rows(q, TK_GATEUP, l, f.hidden);  // each task writes a slice of x_mid[l]
    for (int s = 0; s < n; ++s)
      for (int j = 0; j < (int)d_pl.parts[s].size(); ++j)
        for (int kc = 0; kc < c->ndc; ++kc) {  // K chunks of the same rows run back to back
          Task t = gemv_task(TK_DOWN, l, d_pl, s, j);
          t.aux = (uint16_t)(c->tc ? t.aux : kc);
          add_wait(t, ev_gu(c, l));
          add_notify(t, ev_down(c, l));
          if (tp) t.pad0 = 1;
          evc[ev_down(c, l)] += tp ? (uint32_t)c->tp_ranks : 1u;
          q[s].push_back(t);
        }
  }
  {
    int idx = 0;
    for (int s = 0; s < n; ++s)
      for (int j = 0; j < (int)lm_pl.parts[s].size(); ++j) {
        Task t = gemv_task(TK_LMHEAD, L, lm_pl, s, j);
        add_wait(t, ev_down(c, L - 1));
        if (!c->tc) t.index = (uint32_t)idx;  // argmax partial slot (tensor-core: the tile's)
        ++idx;
        push_static(s, t);
      }
    c->n_lm = c->tc ? c->tc_tiles[TK_LMHEAD] : idx;
    evc[c->ev_lm] = (uint32_t)c->n_lm;
    evc[c->ev_tok] = 1u;
    if (tp) evc[c->ev_lmx] = (uint32_t)(c->tp_ranks * f.max_batch);  // one exchange per rank and sequence
  }
  if (dyn) {
    // every SM ends its step with a static LM-head task (the claim counters of a step are
    // recycled by the token pick, which needs every SM's claims of two steps back done)
    for (int s = 0; s < n; ++s)
      if (q[s].empty() || q[s].back().kind != TK_LMHEAD)
        return fail(c, MK_ERR_UNSUPPORTED, "run-time claims need an LM-head task on every SM");
    // validate the round-robin view with the ordinary checks
    c->g.tasks.clear();
    for (int s = 0; s < n; ++s)
      for (auto& t : qv[s]) c->g.tasks.push_back({t, s});
    if (int rc = validate(c, to_vtasks(c->g), evc)) return rc;
  }
  c->g.tasks.clear();
  c->qbegin.assign(n + 1, 0);
  uint64_t wbytes = 0;
  for (auto& t : pool_tasks) {
    switch (t.kind) {
      case TK_QKV: case TK_OPROJ: case TK_GATEUP: wbytes += (uint64_t)t.nrows * f.hidden * 2; break;
      case TK_DOWN: wbytes += (uint64_t)t.nrows * f.ffn * 2; break;
    }
  }
  for (int s = 0; s < n; ++s) {
    c->qbegin[s] = (uint32_t)c->g.tasks.size();
    for (auto& t : q[s]) {
      c->g.tasks.push_back({t, s});
      if (c->tc) {
        if (is_gemv_kind(t.kind)) wbytes += (uint64_t)t.nrows * kSlotBytes;
        continue;
      }
      switch (t.kind) {
        case TK_QKV: case TK_OPROJ: case TK_GATEUP: case TK_LMHEAD: wbytes += (uint64_t)t.nrows * f.hidden * 2; break;
        case TK_DOWN: {
          const int k0 = t.aux * c->kdc;
          wbytes += (uint64_t)t.nrows * std::min(c->kdc, f.ffn - k0) * 2;
          break;
        }
      }
    }
  }
  c->qbegin[n] = (uint32_t)c->g.tasks.size();
  c->g.ev_count = evc;
  c->g.n_sms = n;
  c->weight_bytes_per_step = wbytes;
  if (dyn) {  // the pools' tasks follow the queues (SM -1: whoever claims them)
    for (auto& fi : c->pool_first) fi += c->qbegin[n];
    for (auto& t : pool_tasks) c->g.tasks.push_back({t, -1});
    return MK_OK;
  }
  if (tp) return MK_OK;  // a shard is validated together with the other ranks (validate_tp)
  return validate(c, to_vtasks(c->g), evc);
}

void layout(mk_ctx* c) {
  const mk_config& f = c->cfg;
  const int L = f.n_layers, H = f.hidden, F = f.ffn, D = f.head_dim, nq = f.n_q_heads, nkv = f.n_kv_heads;
  const int B = f.max_batch;
  // weight arena
  uint64_t o = 0;
  c->loff.resize(L);
  c->off_embed = o;
  o = align256(o + (uint64_t)(c->tp_ranks > 1 ? c->tp_vfull : f.vocab) * H * 2);  // the whole table on every rank
  // bytes of one projection: row-major, or whole kTcRows x kTcUnitK blocks (tensor-core)
  auto mat = [&](int kind, int rows, int K) -> uint64_t {
    if (c->tc) return (uint64_t)c->tc_tiles[kind] * c->tc_nk[kind] * kSlotBytes;
    return (uint64_t)rows * K * 2;
  };
  for (int l = 0; l < L; ++l) {
    LayerOff& lo = c->loff[l];
    lo.qkv = o;
    o = align256(o + mat(TK_QKV, c->rows_qkv, H));
    lo.o = o;
    o = align256(o + mat(TK_OPROJ, H, nq * D));
    lo.gu = o;
    o = align256(o + mat(TK_GATEUP, c->rows_gu, H));
    lo.d = o;
    o = align256(o + mat(TK_DOWN, H, F));
    lo.attn_norm = o;
    o = align256(o + (uint64_t)H * 2);
    lo.mlp_norm = o;
    o = align256(o + (uint64_t)H * 2);
    lo.qkn = o;  // QK-norm gains and biases (0 bytes without QK-norm)
    o = align256(o + (f.qk_norm ? (uint64_t)2 * (nq + nkv) * D * 2 : 0));
  }
  c->off_lm = o;
  o = align256(o + mat(TK_LMHEAD, f.vocab, H));
  c->off_fnorm = o;
  o = align256(o + (uint64_t)H * 2);
  c->arena_bytes = o;
  // workspace
  size_t w = 0;
  auto take = [&](size_t bytes) {
    size_t at = w;
    w = align256(w + bytes);
    return at;
  };
  // room for re-partitioned graphs (mk_set_sm_weights) without changing the workspace size
  c->task_cap = c->g.tasks.size() * 2 + (size_t)c->n_sms * 16;
  c->lm_cap = (size_t)c->n_lm * 2 + (size_t)c->n_sms * 4;
  // run-time claims: queue entries (one per SM and pool) plus pools of up to 4 tasks per SM
  c->pool_cap = 5 * L;  // QKV, attention (priority claims), O, gate/up, down
  c->task_cap = std::max(c->task_cap, c->g.tasks.size() + (size_t)c->n_sms * c->pool_cap * 5);
  c->ws_tasks = take(c->task_cap * sizeof(Task));
  c->ws_pools = take((size_t)c->pool_cap * 2 * sizeof(uint32_t));
  c->pcnt_bytes = (size_t)4 * c->pool_cap * sizeof(uint32_t);
  c->ws_pcnt = take(c->pcnt_bytes);
  c->ws_qbegin = take((c->n_sms + 1) * sizeof(uint32_t));
  c->ws_evcount = take(c->n_events * sizeof(uint32_t));
  c->ev_bytes = c->n_events * sizeof(uint32_t);
  c->ws_ev = take(c->ev_bytes);
  c->acnt_bytes = (size_t)L * B * nkv * sizeof(uint32_t);
  c->ws_acnt = take(c->acnt_bytes);
  c->ws_err = take(4 * sizeof(uint32_t));
  c->ws_loff = take(L * sizeof(LayerOff));
  c->ws_rope = take((size_t)f.max_seq * (D / 2) * sizeof(float2));
  c->ws_xin = take((size_t)(L + 1) * B * H * 4);
  c->ws_xmid = take((size_t)L * B * H * 4);
  c->ws_q = take((size_t)L * B * nq * D * 4);
  c->ws_kraw = take(f.qk_norm ? (size_t)L * B * nkv * D * 4 : 4);
  c->ws_o = take((size_t)L * B * nq * D * 4);
  c->ws_h = take((size_t)L * B * F * 4);
  c->ws_part = take((size_t)L * B * nq * c->nch * (D + 2) * 4);
  c->ws_lmval = take(c->lm_cap * B * 4);
  c->ws_lmidx = take(c->lm_cap * B * 4);
  // tensor-core partial records and tile arrival counters
  c->rec_cap = c->tc ? c->n_recs * 2 + (size_t)c->n_sms * 16 : 0;
  c->ws_tpart = take(std::max<size_t>(c->rec_cap, 1) * kTcRecFloats * 4);
  c->tcnt_bytes = c->tc ? (size_t)L * c->n_tile_ids * sizeof(uint32_t) : 4;
  c->ws_tcnt = take(c->tcnt_bytes);
  // prefill scratch: X, XN, Y, Q, O, HH per row
  const long long ycols = std::max<long long>(std::max(c->rows_qkv, c->rows_gu), H);
  c->pf_rows = (int)std::min<long long>(1024, (long long)B * f.max_seq);
  const long long per_row = (long long)H * 2 + ycols + (long long)nq * D * 2 + F;
  c->ws_pf = take((size_t)c->pf_rows * per_row * 4);
  if (c->tp_ranks > 1) {
    // receive buffers of the row-parallel projections [L][ranks][B][H] and the argmax slots
    c->recv_o_bytes = (size_t)L * c->tp_ranks * B * H * 4;
    c->ws_recv_o = take(c->recv_o_bytes);
    c->ws_recv_d = take(c->recv_o_bytes);
    c->ws_lmx = take((size_t)c->tp_ranks * B * 8);
  }
  c->ws_bytes = w;
  c->kv_bytes = (size_t)L * 2 * B * nkv * f.max_seq * D * 2;
}

int check_config(const mk_config* f, std::string* why) {
  auto bad = [&](const char* m) {
    *why = m;
    return MK_ERR_INVALID_ARG;
  };
  if (!f) return bad("config is NULL");
  if (f->n_layers < 1 || f->n_layers > 1024) return bad("n_layers out of range");
  if (f->hidden < 8 || f->hidden % 8) return bad("hidden must be a positive multiple of 8");
  if (f->ffn < 8 || f->ffn % 8) return bad("ffn must be a positive multiple of 8");
  if (f->head_dim != 64 && f->head_dim != 128) return bad("head_dim must be 64 or 128");
  if (f->n_q_heads < 1 || f->n_kv_heads < 1 || f->n_q_heads % f->n_kv_heads) return bad("bad head counts");
  if (f->n_q_heads / f->n_kv_heads > 4) return bad("more than 4 query heads per KV head");
  if (f->n_q_heads * f->head_dim != f->hidden) return bad("hidden must equal n_q_heads * head_dim");
  if (f->vocab < 2) return bad("vocab too small");
  if (!(f->rms_eps > 0) || !(f->rope_theta > 0)) return bad("rms_eps and rope_theta must be > 0");
  if (f->max_batch < 1 || f->max_batch > MK_MAX_BATCH) return bad("max_batch out of range");
  if (f->max_seq < 1 || f->max_seq > (1 << 20)) return bad("max_seq out of range");
  if (f->tie_embeddings != 0) return bad("tied embeddings are not supported");
  if (f->qk_norm != 0 && f->qk_norm != 1) return bad("qk_norm must be 0 or 1");
  if (f->tc_min_batch != 0 && (f->tc_min_batch < 2 || f->tc_min_batch > kMaxDecodeBatch + 1))
    return bad("tc_min_batch must be 0 or in [2, 5]");
  if (f->hidden > 4 * kSegElems || f->ffn > 8 * kSegElems) return bad("hidden or ffn too large");
  return MK_OK;
}

// RoPE table: cos/sin of pos * theta^(-2i/D), computed in double and rounded to fp32.
void rope_table(const mk_config& f, std::vector<float2>& out) {
  const int half = f.head_dim / 2;
  out.resize((size_t)f.max_seq * half);
  for (int i = 0; i < half; ++i) {
    const double inv = std::pow((double)f.rope_theta, -2.0 * i / f.head_dim);
    for (int p = 0; p < f.max_seq; ++p) {
      const double a = (double)p * inv;
      out[(size_t)p * half + i] = make_float2((float)std::cos(a), (float)std::sin(a));
    }
  }
}

// Tensor-core weight layout of a [rows][K] bf16 matrix (row(i) = pointer to row i): blocks
// of kTcRows x kTcUnitK, block (tile t, K unit u) at (t * nk + u) * kSlotBytes; inside a block,
// core matrix (8-row group g, 8-element K group j) at (g * 16 + j) * 128 bytes and its row r at
// r * 16 bytes.  Rows and K past the matrix are zeros.
template <class RowFn>
void pack_blocks(RowFn row, int rows, int K, std::vector<uint16_t>& out) {
  const int tiles = (rows + kTcRows - 1) / kTcRows, nk = (K + kTcUnitK - 1) / kTcUnitK;
  constexpr int kBlockElems = kTcRows * kTcUnitK;
  out.assign((size_t)tiles * nk * kBlockElems, 0);
  for (int i = 0; i < rows; ++i) {
    const uint16_t* src = row(i);
    const int t = i / kTcRows, g = (i % kTcRows) / 8, r = i % 8;
    for (int k = 0; k < K; k += 8) {
      const int u = k / kTcUnitK, j = (k % kTcUnitK) / 8;
      uint16_t* dst = &out[(size_t)(t * nk + u) * kBlockElems + (size_t)(g * (kTcUnitK / 8) + j) * 64 + r * 8];
      std::memcpy(dst, src + k, (size_t)std::min(8, K - k) * 2);
    }
  }
}

bool cuda_ok(mk_ctx* c, cudaError_t e, const char* what) {
  if (e == cudaSuccess) return true;
  fail(c, MK_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
  return false;
}

// Copy the task graph (tasks, queue offsets, event counts) into the workspace and zero the
// event and arrival counters (the epoch restarts at 1 with the next step).
int upload_graph(mk_ctx* c, uint8_t* W) {
  std::vector<Task> tv;
  for (auto& r : c->g.tasks) tv.push_back(r.t);
  if (!cuda_ok(c, cudaMemcpy(W + c->ws_tasks, tv.data(), tv.size() * sizeof(Task), cudaMemcpyHostToDevice),
               "task upload") ||
      !cuda_ok(c, cudaMemcpy(W + c->ws_qbegin, c->qbegin.data(), c->qbegin.size() * 4, cudaMemcpyHostToDevice),
               "queue upload") ||
      !cuda_ok(c, cudaMemcpy(W + c->ws_evcount, c->g.ev_count.data(), c->g.ev_count.size() * 4,
                             cudaMemcpyHostToDevice),
               "event upload") ||
      !cuda_ok(c, cudaMemset(W + c->ws_ev, 0, c->ev_bytes), "counter reset") ||
      !cuda_ok(c, cudaMemset(W + c->ws_acnt, 0, c->acnt_bytes), "counter reset") ||
      !cuda_ok(c, cudaMemset(W + c->ws_tcnt, 0, c->tcnt_bytes), "counter reset") ||
      !cuda_ok(c, cudaMemset(W + c->ws_pcnt, 0, c->pcnt_bytes), "counter reset"))
    return MK_ERR_CUDA;
  if (!c->pool_first.empty()) {
    std::vector<uint32_t> pl;
    for (size_t p = 0; p < c->pool_first.size(); ++p) {
      pl.push_back(c->pool_first[p]);
      pl.push_back(c->pool_count[p]);
    }
    if (!cuda_ok(c, cudaMemcpy(W + c->ws_pools, pl.data(), pl.size() * 4, cudaMemcpyHostToDevice), "pool upload"))
      return MK_ERR_CUDA;
  }
  c->epoch = 0;
  return MK_OK;
}

// Everything after the config, device and SM count are set: kernel geometry, the task
// graph and the arena / workspace layout.  Tensor-parallel shards also come here (their
// tp_* fields set first).
int init_ctx(mk_ctx* c) {
  const mk_config& f = c->cfg;
  c->G = f.n_q_heads / f.n_kv_heads;
  c->rows_qkv = (f.n_q_heads + 2 * f.n_kv_heads) * f.head_dim;
  c->rows_gu = 2 * f.ffn;
  // split-KV chunks: fill the SMs with (sequence, KV head, chunk) tasks, chunks of >= 16 keys
  {
    int per = std::max(1, c->n_sms / (f.max_batch * f.n_kv_heads));
    int by_len = std::max(1, (f.max_seq + 15) / 16);
    c->nch = std::min(std::min(per, by_len), kMaxChunks);
  }
  // batch width: 1; or 4 (sequences beyond the active batch masked), where the down
  // projection runs in K chunks of kDownChunk so its activations fit in registers; or, for
  // more than 4 sequences, kTcBatch on the tensor cores
  {
    const int tc_min = f.tc_min_batch ? f.tc_min_batch : kTcMinBatchDefault;
    c->bm = (f.max_batch >= tc_min) ? kTcBatch : (f.max_batch > 1) ? 4 : 1;
  }
  c->tc = c->bm == kTcBatch;
  c->task_rows = c->tc ? kTcUnitsMax : kTaskRows / c->bm;
  c->kdc = (c->bm == 4) ? std::min(f.ffn, kDownChunk) : f.ffn;
  c->ndc = (f.ffn + c->kdc - 1) / c->kdc;
  c->nseg_h = (f.hidden + kSegElems - 1) / kSegElems;
  c->nseg_f = (c->kdc + kSegElems - 1) / kSegElems;
  c->rps_h = pow2_floor(std::min(kRpsMax, kSlotBytes / (f.hidden * 2)));
  c->rps_f = pow2_floor(std::min(kRpsMax, kSlotBytes / (c->kdc * 2)));
  // the GEMV takes every segment but the last of a K chunk as full
  const bool ragged_chunk = c->ndc > 1 && f.ffn - (c->ndc - 1) * c->kdc < (c->nseg_f - 1) * kSegElems;
  if (!c->tc && ((f.max_batch == 1 && f.ffn * 2 > kSlotBytes) || f.hidden * 2 > kSlotBytes || ragged_chunk))
    return fail(c, MK_ERR_UNSUPPORTED, "a weight row does not fit one ring stage");
  if (c->tc) {
    // tiles of kTcRows rows, K in units of kTcUnitK (rows and K past the end are zero padding)
    const int H = f.hidden;
    auto set = [&](int kind, int rows, int K) {
      c->tc_tiles[kind] = (rows + kTcRows - 1) / kTcRows;
      c->tc_nk[kind] = (K + kTcUnitK - 1) / kTcUnitK;
    };
    set(TK_QKV, c->rows_qkv, H);
    set(TK_OPROJ, H, f.n_q_heads * f.head_dim);
    set(TK_GATEUP, c->rows_gu, H);
    set(TK_DOWN, H, f.ffn);
    set(TK_LMHEAD, f.vocab, H);
    int base = 0;
    for (int k : {TK_QKV, TK_OPROJ, TK_GATEUP, TK_DOWN, TK_LMHEAD}) {
      c->tc_tile_base[k] = base;
      base += c->tc_tiles[k];
    }
    c->n_tile_ids = base;
    c->variant = find_decode_variant(0, 1, 0, 1, f.head_dim, kTcBatch, f.qk_norm, 0);
  } else {
    c->variant = find_decode_variant(c->nseg_h, c->rps_h, c->nseg_f, c->rps_f, f.head_dim, c->bm, f.qk_norm, 0,
                                     c->tp_ranks > 1 ? 1 : 0);
  }
  c->sm_weights.assign(c->n_sms, 1.0);
  if (int rc = build_graph(c)) return rc;
  layout(c);
  c->pos.assign(f.max_batch, 0);
  return MK_OK;
}

}  // namespace

namespace mk {
TensorMapEncodeFn get_tensor_map_encoder() {
  static TensorMapEncodeFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<TensorMapEncodeFn>(p);
  }
  return fn;
}
}  // namespace mk


namespace {
// Emulated tensor parallel: each rank's shard of the host weights (heads, ffn rows, vocab rows;
// the O and down projections' column slices copied out), loaded into its arena and workspace
// regions; then every rank's queues into the combined arrays the kernel walks.
int tp_load_weights(mk_ctx* c, const mk_host_weights* w, void* weight_arena, void* workspace, void* stream) {
  const mk_config& f = c->cfg;
  const int R = c->tp_ranks, L = f.n_layers, H = f.hidden, D = f.head_dim;
  const int nq_l = f.n_q_heads / R, nkv_l = f.n_kv_heads / R, F_l = f.ffn / R, V_l = f.vocab / R;
  if (!w->embed || !w->lm_head || !w->final_norm || !w->attn_norm || !w->wq || !w->wk || !w->wv || !w->wo ||
      !w->mlp_norm || !w->wg || !w->wu || !w->wd)
    return fail(c, MK_ERR_INVALID_ARG, "a weight pointer is NULL");
  if ((reinterpret_cast<uintptr_t>(weight_arena) | reinterpret_cast<uintptr_t>(workspace)) & 255)
    return fail(c, MK_ERR_INVALID_ARG, "arena and workspace must be 256-byte aligned");
  uint8_t* A = static_cast<uint8_t*>(weight_arena);
  uint8_t* W = static_cast<uint8_t*>(workspace);
  for (int r = 0; r < R; ++r) {
    std::vector<const uint16_t*> wq(L), wk(L), wv(L), wo(L), wg(L), wu(L), wd(L);
    std::vector<std::vector<uint16_t>> wo_s(L), wd_s(L);
    for (int l = 0; l < L; ++l) {
      if (!w->wq[l] || !w->wk[l] || !w->wv[l] || !w->wo[l] || !w->wg[l] || !w->wu[l] || !w->wd[l])
        return fail(c, MK_ERR_INVALID_ARG, "a per-layer weight pointer is NULL");
      wq[l] = w->wq[l] + (size_t)r * nq_l * D * H;   // rows of this rank's query heads
      wk[l] = w->wk[l] + (size_t)r * nkv_l * D * H;  // ... KV heads
      wv[l] = w->wv[l] + (size_t)r * nkv_l * D * H;
      wg[l] = w->wg[l] + (size_t)r * F_l * H;        // ffn rows
      wu[l] = w->wu[l] + (size_t)r * F_l * H;
      wo_s[l].resize((size_t)H * nq_l * D);          // columns of this rank's heads
      wd_s[l].resize((size_t)H * F_l);               // columns of its ffn rows
      for (int i = 0; i < H; ++i) {
        std::memcpy(&wo_s[l][(size_t)i * nq_l * D], w->wo[l] + (size_t)i * f.n_q_heads * D + (size_t)r * nq_l * D,
                    (size_t)nq_l * D * 2);
        std::memcpy(&wd_s[l][(size_t)i * F_l], w->wd[l] + (size_t)i * f.ffn + (size_t)r * F_l, (size_t)F_l * 2);
      }
      wo[l] = wo_s[l].data();
      wd[l] = wd_s[l].data();
    }
    mk_host_weights hw = *w;
    hw.lm_head = w->lm_head + (size_t)r * V_l * H;  // this rank's vocab rows; the embedding stays whole
    hw.wq = wq.data();
    hw.wk = wk.data();
    hw.wv = wv.data();
    hw.wo = wo.data();
    hw.wg = wg.data();
    hw.wu = wu.data();
    hw.wd = wd.data();
    mk_ctx* sh = c->tp_shards[r];
    if (int rc = mk_load_weights(sh, &hw, A + c->tp_arena_off[r], W + c->tp_ws_off[r], stream))
      return fail(c, rc, "rank " + std::to_string(r) + ": " + sh->err);
  }
  if (!cuda_ok(c, cudaMemcpy(W + c->tp_ws_tasks, c->tp_tasks.data(), c->tp_tasks.size() * sizeof(Task),
                             cudaMemcpyHostToDevice), "task upload") ||
      !cuda_ok(c, cudaMemcpy(W + c->tp_ws_qbegin, c->tp_qbegin.data(), c->tp_qbegin.size() * 4,
                             cudaMemcpyHostToDevice), "queue upload"))
    return MK_ERR_CUDA;
  c->arena = A;
  c->ws = W;
  c->loaded = true;
  c->epoch = 0;
  return MK_OK;
}

// Every rank's counters back to zero (the epoch restarts); the error word is rank 0's.
int tp_reset_counters(mk_ctx* c) {
  for (mk_ctx* sh : c->tp_shards)
    if (!cuda_ok(c, cudaMemset(sh->ws + sh->ws_ev, 0, sh->ev_bytes), "counter reset") ||
        !cuda_ok(c, cudaMemset(sh->ws + sh->ws_acnt, 0, sh->acnt_bytes), "counter reset") ||
        !cuda_ok(c, cudaMemset(sh->ws + sh->ws_err, 0, 16), "error reset"))
      return MK_ERR_CUDA;
  if (!cuda_ok(c, cudaDeviceSynchronize(), "reset sync")) return MK_ERR_CUDA;
  c->epoch = 0;
  return MK_OK;
}

int tp_sync_status(mk_ctx* c) {
  mk_ctx* s0 = c->tp_shards[0];
  uint32_t e[4];
  if (!cuda_ok(c, cudaMemcpy(e, s0->ws + s0->ws_err, 16, cudaMemcpyDeviceToHost), "error read")) return MK_ERR_CUDA;
  if (e[ERR_CODE] == 0) return MK_OK;
  if (e[ERR_CODE] == DEV_ERR_BAD_TOKEN && e[ERR_ABORT] == 0) {
    cudaMemset(s0->ws + s0->ws_err, 0, 16);
    return fail(c, MK_ERR_INVALID_ARG, "a token id was outside [0, vocab); row 0 was used");
  }
  char buf[160];
  snprintf(buf, sizeof buf, "device wait timed out (kind %u, at %u, task %u)", e[ERR_CODE], e[ERR_WHERE], e[ERR_TASK]);
  if (int rc = tp_reset_counters(c)) return rc;
  return fail(c, MK_ERR_DEVICE_TIMEOUT, buf);
}
}  // namespace
// =========================================================================================
extern "C" {

int mk_build_taskgraph(const mk_config* cfg, int device, mk_ctx** out) {
  if (!out) return fail(nullptr, MK_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  std::string why;
  int rc = check_config(cfg, &why);
  if (rc) return fail(nullptr, rc, why);
  mk_ctx* c = new mk_ctx();
  c->cfg = *cfg;
  c->device = device;
  if (device >= 0) {
    int n = 0;
    cudaError_t e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device);
    if (e != cudaSuccess) {
      delete c;
      return fail(nullptr, MK_ERR_CUDA, std::string("cudaDeviceGetAttribute: ") + cudaGetErrorString(e));
    }
    c->n_sms = n;
  } else {
    c->n_sms = 148;  // planning without a device: a B200's SM count
  }
  rc = init_ctx(c);
  if (rc) {
    std::string m = c->err;
    delete c;
    return fail(nullptr, rc, m);
  }
  *out = c;
  return MK_OK;
}

size_t mk_weight_arena_bytes(const mk_ctx* c) { return c ? c->arena_bytes : 0; }
size_t mk_workspace_bytes(const mk_ctx* c) { return c ? c->ws_bytes : 0; }
size_t mk_kv_cache_bytes(const mk_ctx* c) { return c ? c->kv_bytes : 0; }

int mk_load_weights(mk_ctx* c, const mk_host_weights* w, void* weight_arena, void* workspace, void* stream) {
  if (!c) return fail(nullptr, MK_ERR_INVALID_ARG, "ctx is NULL");
  if (!w || !weight_arena || !workspace) return fail(c, MK_ERR_INVALID_ARG, "NULL weights or buffers");
  if (!c->tp_shards.empty()) return tp_load_weights(c, w, weight_arena, workspace, stream);
  if (c->device < 0) return fail(c, MK_ERR_STATE, "context was planned without a device");
  if ((reinterpret_cast<uintptr_t>(weight_arena) | reinterpret_cast<uintptr_t>(workspace)) & 255)
    return fail(c, MK_ERR_INVALID_ARG, "arena and workspace must be 256-byte aligned");
  const mk_config& f = c->cfg;
  const int L = f.n_layers, H = f.hidden, F = f.ffn, D = f.head_dim, nq = f.n_q_heads, nkv = f.n_kv_heads;
  if (!w->embed || !w->lm_head || !w->final_norm || !w->attn_norm || !w->wq || !w->wk || !w->wv || !w->wo ||
      !w->mlp_norm || !w->wg || !w->wu || !w->wd)
    return fail(c, MK_ERR_INVALID_ARG, "a weight pointer is NULL");
  for (int l = 0; l < L; ++l)
    if (!w->attn_norm[l] || !w->wq[l] || !w->wk[l] || !w->wv[l] || !w->wo[l] || !w->mlp_norm[l] || !w->wg[l] ||
        !w->wu[l] || !w->wd[l])
      return fail(c, MK_ERR_INVALID_ARG, "a per-layer weight pointer is NULL");
  if (f.qk_norm) {
    if (!w->q_norm_w || !w->q_norm_b || !w->k_norm_w || !w->k_norm_b)
      return fail(c, MK_ERR_INVALID_ARG, "a QK-norm model needs q_norm_w, q_norm_b, k_norm_w and k_norm_b");
    for (int l = 0; l < L; ++l)
      if (!w->q_norm_w[l] || !w->q_norm_b[l] || !w->k_norm_w[l] || !w->k_norm_b[l])
        return fail(c, MK_ERR_INVALID_ARG, "a per-layer QK-norm pointer is NULL");
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (!cuda_ok(c, cudaSetDevice(c->device), "cudaSetDevice")) return MK_ERR_CUDA;
  uint8_t* A = static_cast<uint8_t*>(weight_arena);
  auto put = [&](uint64_t off, const void* src, size_t bytes) {
    return cuda_ok(c, cudaMemcpyAsync(A + off, src, bytes, cudaMemcpyHostToDevice, s), "weight copy");
  };
  // tensor-core layout: each projection re-laid in blocks, copied synchronously (staging reused)
  std::vector<uint16_t> blk;
  auto put_blocks = [&](uint64_t off, const uint16_t* base, size_t stride, int rows, int K) {
    pack_blocks([&](int i) { return base + (size_t)i * stride; }, rows, K, blk);
    return cuda_ok(c, cudaMemcpy(A + off, blk.data(), blk.size() * 2, cudaMemcpyHostToDevice), "weight copy");
  };
  if (!put(c->off_embed, w->embed, (size_t)(c->tp_ranks > 1 ? c->tp_vfull : f.vocab) * H * 2)) return MK_ERR_CUDA;
  if (c->tc ? !put_blocks(c->off_lm, w->lm_head, H, f.vocab, H) : !put(c->off_lm, w->lm_head, (size_t)f.vocab * H * 2))
    return MK_ERR_CUDA;
  if (!put(c->off_fnorm, w->final_norm, (size_t)H * 2)) return MK_ERR_CUDA;
  std::vector<uint16_t> qkv((size_t)c->rows_qkv * H), gu((size_t)c->rows_gu * H);
  const int G = c->G, half = D / 2;
  for (int l = 0; l < L; ++l) {
    // QKV rows grouped per KV head g: [q heads g*G.., k head g, v head g]; q and k rows of a
    // head in RoPE pairs (i, i + D/2) -> packed (2i, 2i + 1); v rows in natural order
    size_t r = 0;
    auto copy_row = [&](const uint16_t* src, int row) {
      std::memcpy(&qkv[r * H], src + (size_t)row * H, (size_t)H * 2);
      ++r;
    };
    for (int g = 0; g < nkv; ++g) {
      for (int hq = g * G; hq < (g + 1) * G; ++hq)
        for (int i = 0; i < half; ++i) {
          copy_row(w->wq[l], hq * D + i);
          copy_row(w->wq[l], hq * D + i + half);
        }
      for (int i = 0; i < half; ++i) {
        copy_row(w->wk[l], g * D + i);
        copy_row(w->wk[l], g * D + i + half);
      }
      for (int i = 0; i < D; ++i) copy_row(w->wv[l], g * D + i);
    }
    for (int i = 0; i < F; ++i) {
      std::memcpy(&gu[(size_t)(2 * i) * H], w->wg[l] + (size_t)i * H, (size_t)H * 2);
      std::memcpy(&gu[(size_t)(2 * i + 1) * H], w->wu[l] + (size_t)i * H, (size_t)H * 2);
    }
    const LayerOff& lo = c->loff[l];
    if (f.qk_norm) {
      const size_t qb = (size_t)nq * D * 2, kb = (size_t)nkv * D * 2;
      if (!put(lo.qkn, w->q_norm_w[l], qb) || !put(lo.qkn + qb, w->q_norm_b[l], qb) ||
          !put(lo.qkn + 2 * qb, w->k_norm_w[l], kb) || !put(lo.qkn + 2 * qb + kb, w->k_norm_b[l], kb))
        return MK_ERR_CUDA;
    }
    if (c->tc) {
      if (!put_blocks(lo.qkv, qkv.data(), H, c->rows_qkv, H) || !put_blocks(lo.o, w->wo[l], nq * D, H, nq * D) ||
          !put_blocks(lo.gu, gu.data(), H, c->rows_gu, H) || !put_blocks(lo.d, w->wd[l], F, H, F) ||
          !put(lo.attn_norm, w->attn_norm[l], (size_t)H * 2) || !put(lo.mlp_norm, w->mlp_norm[l], (size_t)H * 2) ||
          !cuda_ok(c, cudaStreamSynchronize(s), "weight copy"))
        return MK_ERR_CUDA;
      continue;
    }
    // synchronous copies: the staging vectors are reused for the next layer
    if (!cuda_ok(c, cudaMemcpy(A + lo.qkv, qkv.data(), qkv.size() * 2, cudaMemcpyHostToDevice), "qkv copy"))
      return MK_ERR_CUDA;
    if (!cuda_ok(c, cudaMemcpy(A + lo.gu, gu.data(), gu.size() * 2, cudaMemcpyHostToDevice), "gate/up copy"))
      return MK_ERR_CUDA;
    if (c->ndc > 1) {
      // W_down chunk-major: chunk k holds columns [k*kdc, k*kdc + kc) of every row, contiguous
      std::vector<uint16_t> dk((size_t)H * c->kdc);
      for (int k = 0; k < c->ndc; ++k) {
        const int k0 = k * c->kdc, kc = std::min(c->kdc, F - k0);
        for (int r = 0; r < H; ++r)
          std::memcpy(&dk[(size_t)r * kc], w->wd[l] + (size_t)r * F + k0, (size_t)kc * 2);
        if (!cuda_ok(c, cudaMemcpy(A + lo.d + (size_t)H * k0 * 2, dk.data(), (size_t)H * kc * 2,
                                   cudaMemcpyHostToDevice),
                     "down chunk copy"))
          return MK_ERR_CUDA;
      }
    } else if (!put(lo.d, w->wd[l], (size_t)H * F * 2)) {
      return MK_ERR_CUDA;
    }
    if (!put(lo.o, w->wo[l], (size_t)H * nq * D * 2) ||
        !put(lo.attn_norm, w->attn_norm[l], (size_t)H * 2) || !put(lo.mlp_norm, w->mlp_norm[l], (size_t)H * 2))
      return MK_ERR_CUDA;
  }
  // workspace: task graph, counts, zeroed counters, offsets, RoPE table
  uint8_t* W = static_cast<uint8_t*>(workspace);
  std::vector<float2> rope;
  rope_table(f, rope);
  if (upload_graph(c, W) != MK_OK) return MK_ERR_CUDA;
  if (!cuda_ok(c, cudaMemcpy(W + c->ws_loff, c->loff.data(), c->loff.size() * sizeof(LayerOff),
                             cudaMemcpyHostToDevice),
               "offset upload") ||
      !cuda_ok(c, cudaMemcpy(W + c->ws_rope, rope.data(), rope.size() * sizeof(float2), cudaMemcpyHostToDevice),
               "rope upload") ||
      !cuda_ok(c, cudaMemset(W + c->ws_ev, 0, c->ev_bytes), "counter reset") ||
      !cuda_ok(c, cudaMemset(W + c->ws_acnt, 0, c->acnt_bytes), "counter reset") ||
      !cuda_ok(c, cudaMemset(W + c->ws_tcnt, 0, c->tcnt_bytes), "counter reset") ||
      !cuda_ok(c, cudaMemset(W + c->ws_pcnt, 0, c->pcnt_bytes), "counter reset") ||
      !cuda_ok(c, cudaMemset(W + c->ws_err, 0, 16), "error reset") ||
      !cuda_ok(c, cudaStreamSynchronize(s), "load sync"))
    return MK_ERR_CUDA;
  c->arena = A;
  c->ws = W;
  c->loaded = true;
  c->epoch = 0;
  return MK_OK;
}

int mk_prefill(mk_ctx* c, const int32_t* tokens, int B, int T, void* kv_cache, float* last_logits, void* stream) {
  if (!c) return fail(nullptr, MK_ERR_INVALID_ARG, "ctx is NULL");
  if (!c->tp_shards.empty())
    return fail(c, MK_ERR_UNSUPPORTED, "tensor-parallel contexts take the prompt as decode steps (or a filled cache)");
  if (!c->loaded) return fail(c, MK_ERR_STATE, "weights not loaded");
  if (!tokens || !kv_cache) return fail(c, MK_ERR_INVALID_ARG, "NULL tokens or cache");
  if (B < 1 || B > c->cfg.max_batch || T < 1 || T > c->cfg.max_seq)
    return fail(c, MK_ERR_INVALID_ARG, "B or T out of range");
  const mk_config& f = c->cfg;
  PrefillParams p;
  p.arena = c->arena;
  p.loff_host = c->loff.data();
  p.off_embed = c->off_embed;
  p.off_lm = c->off_lm;
  p.off_fnorm = c->off_fnorm;
  p.rope = reinterpret_cast<const float2*>(c->ws + c->ws_rope);
  p.kv = static_cast<uint16_t*>(kv_cache);
  const long long ycols = std::max<long long>(std::max(c->rows_qkv, c->rows_gu), f.hidden);
  float* base = reinterpret_cast<float*>(c->ws + c->ws_pf);
  const size_t R = (size_t)c->pf_rows;
  p.X = base;
  p.XN = p.X + R * f.hidden;
  p.Y = p.XN + R * f.hidden;
  p.Q = p.Y + R * ycols;
  p.O = p.Q + R * f.n_q_heads * f.head_dim;
  p.HH = p.O + R * f.n_q_heads * f.head_dim;
  p.rows_cap = c->pf_rows;
  p.H = f.hidden;
  p.nq = f.n_q_heads;
  p.nkv = f.n_kv_heads;
  p.D = f.head_dim;
  p.F = f.ffn;
  p.V = f.vocab;
  p.L = f.n_layers;
  p.max_seq = f.max_seq;
  p.max_batch = f.max_batch;
  p.eps = f.rms_eps;
  p.attn_scale = 1.0f / std::sqrt((float)f.head_dim);
  p.kdc = c->kdc;
  p.ndc = c->ndc;
  p.blocked = c->tc ? 1 : 0;
  p.qk_norm = f.qk_norm;
  std::string err;
  int rc = run_prefill(p, tokens, B, T, last_logits, reinterpret_cast<cudaStream_t>(stream), &err);
  if (rc) return fail(c, rc, err);
  c->B = B;
  for (int b = 0; b < B; ++b) c->pos[b] = T;
  return MK_OK;
}

int mk_set_positions(mk_ctx* c, const int32_t* host_pos, int B) {
  if (!c) return fail(nullptr, MK_ERR_INVALID_ARG, "ctx is NULL");
  if (!host_pos || B < 1 || B > c->cfg.max_batch) return fail(c, MK_ERR_INVALID_ARG, "bad positions");
  for (int b = 0; b < B; ++b)
    if (host_pos[b] < 0 || host_pos[b] >= c->cfg.max_seq) return fail(c, MK_ERR_INVALID_ARG, "position out of range");
  c->B = B;
  for (int b = 0; b < B; ++b) c->pos[b] = host_pos[b];
  return MK_OK;
}

int mk_get_positions(const mk_ctx* c, int32_t* host_pos, int capacity) {
  if (!c || (capacity > 0 && !host_pos)) return MK_ERR_INVALID_ARG;
  for (int b = 0; b < c->B && b < capacity; ++b) host_pos[b] = c->pos[b];
  return c->B;
}

namespace {
// The kernel's view of context c (a whole model, or one tensor-parallel shard) for a launch of
// n_steps decode steps; `run` holds the positions, active batch, epoch and test settings.
void make_params(const mk_ctx* c, const mk_ctx* run, const int32_t* tokens, int n_steps, void* kv_cache,
                 float* logits, int32_t* next_tokens, DecodeParams& P) {
  const mk_config& f = c->cfg;
  std::memset(&P, 0, sizeof(P));
  uint8_t* W = c->ws;
  P.tasks = reinterpret_cast<const Task*>(W + c->ws_tasks);
  P.qbegin = reinterpret_cast<const uint32_t*>(W + c->ws_qbegin);
  P.ev_count = reinterpret_cast<const uint32_t*>(W + c->ws_evcount);
  P.ev = reinterpret_cast<uint32_t*>(W + c->ws_ev);
  P.acnt = reinterpret_cast<uint32_t*>(W + c->ws_acnt);
  P.err = reinterpret_cast<uint32_t*>(W + c->ws_err);
  P.arena = c->arena;
  P.loff = reinterpret_cast<const LayerOff*>(W + c->ws_loff);
  P.off_embed = c->off_embed;
  P.off_lm = c->off_lm;
  P.off_fnorm = c->off_fnorm;
  P.rope = reinterpret_cast<const float2*>(W + c->ws_rope);
  P.kv = static_cast<uint16_t*>(kv_cache);
  P.x_in = reinterpret_cast<float*>(W + c->ws_xin);
  P.x_mid = reinterpret_cast<float*>(W + c->ws_xmid);
  P.qbuf = reinterpret_cast<float*>(W + c->ws_q);
  P.kraw = reinterpret_cast<float*>(W + c->ws_kraw);
  P.pools = reinterpret_cast<const uint2*>(W + c->ws_pools);
  P.pcnt = reinterpret_cast<uint32_t*>(W + c->ws_pcnt);
  P.n_pools = (int)c->pool_first.size();
  P.dyn = c->dyn;
  P.qk_norm = f.qk_norm;
  P.obuf = reinterpret_cast<float*>(W + c->ws_o);
  P.hbuf = reinterpret_cast<float*>(W + c->ws_h);
  P.part = reinterpret_cast<float*>(W + c->ws_part);
  P.lm_val = reinterpret_cast<float*>(W + c->ws_lmval);
  P.lm_idx = reinterpret_cast<int32_t*>(W + c->ws_lmidx);
  P.tokens = tokens;
  P.logits = logits;
  P.next_tokens = next_tokens;
  for (int b = 0; b < run->B; ++b) P.pos[b] = run->pos[b];
  P.B = f.max_batch;  // buffer strides use the capacity; the kernel serves sequence 0.. of it
  P.H = f.hidden;
  P.nq = f.n_q_heads;
  P.nkv = f.n_kv_heads;
  P.D = f.head_dim;
  P.F = f.ffn;
  P.V = f.vocab;
  P.L = f.n_layers;
  P.nch = c->nch;
  P.max_seq = f.max_seq;
  P.max_batch = f.max_batch;
  P.n_lm = c->n_lm;
  P.eps = f.rms_eps;
  P.attn_scale = 1.0f / std::sqrt((float)f.head_dim);
  P.nb = run->B;
  P.kdc = c->kdc;
  P.ndc = c->ndc;
  P.tpart = reinterpret_cast<float*>(W + c->ws_tpart);
  P.tcnt = reinterpret_cast<uint32_t*>(W + c->ws_tcnt);
  P.epoch = run->epoch + 1;
  P.ev_lm = (uint32_t)c->ev_lm;
  P.ev_tok = (uint32_t)c->ev_tok;
  P.n_steps = n_steps;
  P.drop_event = run->drop_event;
  P.timeout_ns = run->timeout_ns;
  P.trace = run->trace;
  P.l2_ahead = c->dyn ? 0 : run->l2_ahead;  // the lookahead walks static queues only
  P.min_chunk_keys = run->min_chunk_keys;
  P.head_keys = run->head_keys;
  P.tp_ranks = 1;
}

int tp_decode_launch(mk_ctx* c, const int32_t* tokens, int n_steps, void* kv_cache, float* logits,
                     int32_t* next_tokens, void* stream);

// One launch of the persistent kernel running n_steps greedy decode steps.
int decode_launch(mk_ctx* c, const int32_t* tokens, int n_steps, void* kv_cache, float* logits,
                  int32_t* next_tokens, void* stream) {
  if (!c) return fail(nullptr, MK_ERR_INVALID_ARG, "ctx is NULL");
  if (!c->loaded) return fail(c, MK_ERR_STATE, "weights not loaded");
  if (c->B < 1) return fail(c, MK_ERR_STATE, "no active batch (call mk_prefill or mk_set_positions)");
  if (!tokens || !kv_cache || !logits) return fail(c, MK_ERR_INVALID_ARG, "NULL tokens, cache or logits");
  if (n_steps < 1 || n_steps > MK_MAX_STEPS) return fail(c, MK_ERR_INVALID_ARG, "n_steps out of range");
  if (n_steps > 1 && !next_tokens) return fail(c, MK_ERR_INVALID_ARG, "a multi-step launch needs tokens_out");
  if (c->variant < 0 || c->B > c->bm)
    return fail(c, MK_ERR_UNSUPPORTED, "no decode kernel instantiation for this shape / batch");
  const mk_config& f = c->cfg;
  for (int b = 0; b < c->B; ++b)
    if (c->pos[b] + n_steps > f.max_seq) return fail(c, MK_ERR_INVALID_ARG, "sequence is full (max_seq reached)");
  if (!c->tp_shards.empty()) return tp_decode_launch(c, tokens, n_steps, kv_cache, logits, next_tokens, stream);
  DecodeParams P;
  make_params(c, c, tokens, n_steps, kv_cache, logits, next_tokens, P);
  std::string err;
  int rc = launch_decode(c->variant, P, c->n_sms, reinterpret_cast<cudaStream_t>(stream), &err);
  if (rc) return fail(c, rc, err);
  c->epoch += (uint32_t)n_steps;
  for (int b = 0; b < c->B; ++b) c->pos[b] += n_steps;
  return MK_OK;
}

// Emulated tensor parallel: one launch, every rank's view (see mk_build_taskgraph_tp).
int tp_decode_launch(mk_ctx* c, const int32_t* tokens, int n_steps, void* kv_cache, float* logits,
                     int32_t* next_tokens, void* stream) {
  const int R = c->tp_ranks;
  DecodeParams views[kMaxTpRanks];
  for (int r = 0; r < R; ++r) {
    const mk_ctx* sh = c->tp_shards[r];
    DecodeParams& P = views[r];
    make_params(sh, c, tokens, n_steps, static_cast<uint8_t*>(kv_cache) + c->tp_kv_off[r], logits, next_tokens, P);
    P.tasks = reinterpret_cast<const Task*>(c->ws + c->tp_ws_tasks);  // every rank's queues
    P.qbegin = reinterpret_cast<const uint32_t*>(c->ws + c->tp_ws_qbegin);
    P.err = reinterpret_cast<uint32_t*>(c->tp_shards[0]->ws + c->tp_shards[0]->ws_err);  // one error word
    P.trace = nullptr;
    P.tp_rank = r;
    P.tp_ranks = R;
    P.tp_vbase = sh->tp_vbase;
    P.tp_vfull = sh->tp_vfull;
    P.ev_lmx = (uint32_t)sh->ev_lmx;
    for (int d = 0; d < R; ++d) {
      mk_ctx* pd = c->tp_shards[d];
      P.tp_recv_o[d] = reinterpret_cast<float*>(pd->ws + pd->ws_recv_o);
      P.tp_recv_d[d] = reinterpret_cast<float*>(pd->ws + pd->ws_recv_d);
      P.tp_ev[d] = reinterpret_cast<uint32_t*>(pd->ws + pd->ws_ev);
      P.tp_lmx[d] = reinterpret_cast<uint64_t*>(pd->ws + pd->ws_lmx);
    }
  }
  std::string err;
  int rc = launch_decode_tp(c->variant, views, R, c->tp_sms, reinterpret_cast<cudaStream_t>(stream), &err);
  if (rc) return fail(c, rc, err);
  c->epoch += (uint32_t)n_steps;
  for (int b = 0; b < c->B; ++b) c->pos[b] += n_steps;
  return MK_OK;
}
}  // namespace

int mk_decode_step(mk_ctx* c, const int32_t* tokens, void* kv_cache, float* logits, int32_t* next_tokens,
                   void* stream) {
  return decode_launch(c, tokens, 1, kv_cache, logits, next_tokens, stream);
}

int mk_decode_steps(mk_ctx* c, const int32_t* tokens, int n_steps, void* kv_cache, float* logits,
                    int32_t* tokens_out, void* stream) {
  return decode_launch(c, tokens, n_steps, kv_cache, logits, tokens_out, stream);
}

int mk_sync_status(mk_ctx* c, void* stream) {
  if (!c) return fail(nullptr, MK_ERR_INVALID_ARG, "ctx is NULL");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (!cuda_ok(c, cudaStreamSynchronize(s), "stream sync")) return MK_ERR_CUDA;
  if (!c->loaded) return MK_OK;
  if (!c->tp_shards.empty()) return tp_sync_status(c);
  uint32_t e[4];
  if (!cuda_ok(c, cudaMemcpy(e, c->ws + c->ws_err, 16, cudaMemcpyDeviceToHost), "error read")) return MK_ERR_CUDA;
  if (e[ERR_CODE] == 0) return MK_OK;
  if (e[ERR_CODE] == DEV_ERR_BAD_TOKEN && e[ERR_ABORT] == 0) {
    cudaMemset(c->ws + c->ws_err, 0, 16);
    return fail(c, MK_ERR_INVALID_ARG, "a token id was outside [0, vocab); row 0 was used");
  }
  char buf[160];
  snprintf(buf, sizeof buf, "device wait timed out (kind %u, at %u, task %u)", e[ERR_CODE], e[ERR_WHERE],
           e[ERR_TASK]);
  // reset counters so the context stays usable
  if (!cuda_ok(c, cudaMemset(c->ws + c->ws_ev, 0, c->ev_bytes), "counter reset") ||
      !cuda_ok(c, cudaMemset(c->ws + c->ws_acnt, 0, c->acnt_bytes), "counter reset") ||
      !cuda_ok(c, cudaMemset(c->ws + c->ws_tcnt, 0, c->tcnt_bytes), "counter reset") ||
      !cuda_ok(c, cudaMemset(c->ws + c->ws_pcnt, 0, c->pcnt_bytes), "counter reset") ||
      !cuda_ok(c, cudaMemset(c->ws + c->ws_err, 0, 16), "error reset") ||
      !cuda_ok(c, cudaDeviceSynchronize(), "reset sync"))
    return MK_ERR_CUDA;
  c->epoch = 0;
  return fail(c, MK_ERR_DEVICE_TIMEOUT, buf);
}

int mk_set_wait_timeout_ns(mk_ctx* c, uint64_t ns) {
  if (!c || ns == 0) return fail(c, MK_ERR_INVALID_ARG, "timeout must be > 0");
  c->timeout_ns = ns;
  return MK_OK;
}

int mk_debug_drop_notify(mk_ctx* c, int event_id, int on) {
  if (!c || event_id < 0 || event_id >= c->n_events) return fail(c, MK_ERR_INVALID_ARG, "bad event id");
  c->drop_event = on ? event_id : -1;
  return MK_OK;
}

namespace {
// Re-partition with new per-SM weights for one projection kind (op > 0) or for all (op = 0).
int set_weights(mk_ctx* c, int op, const float* weights, int n, void* stream) {
  if (!c) return fail(nullptr, MK_ERR_INVALID_ARG, "ctx is NULL");
  if (!c->tp_shards.empty()) return fail(c, MK_ERR_UNSUPPORTED, "tensor-parallel graphs keep equal rows per SM");
  if (op != 0 && op != TK_QKV && op != TK_OPROJ && op != TK_GATEUP && op != TK_DOWN && op != TK_LMHEAD)
    return fail(c, MK_ERR_INVALID_ARG, "op must be 0 or a projection task kind");
  if (!weights || n != c->n_sms) return fail(c, MK_ERR_INVALID_ARG, "need one weight per SM");
  std::vector<double> w(n);
  for (int i = 0; i < n; ++i) {
    if (!(weights[i] > 0.f) || !std::isfinite(weights[i]) || weights[i] > 1e3f)
      return fail(c, MK_ERR_INVALID_ARG, "weights must be finite and in (0, 1000]");
    w[i] = weights[i];
  }
  if (c->loaded && !cuda_ok(c, cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)), "stream sync"))
    return MK_ERR_CUDA;
  std::vector<double> old = c->sm_weights;
  std::vector<double> old_op[8];
  for (int k = 0; k < 8; ++k) old_op[k] = c->op_weights[k];
  Graph old_g = c->g;
  std::vector<uint32_t> old_q = c->qbegin;
  const int old_lm = c->n_lm;
  const size_t old_recs = c->n_recs;
  const uint64_t old_wb = c->weight_bytes_per_step;
  if (op == 0) {
    c->sm_weights = w;
    for (int k = 0; k < 8; ++k) c->op_weights[k].clear();
  } else {
    c->op_weights[op] = w;
  }
  int rc = build_graph(c);
  if (rc == MK_OK && (c->g.tasks.size() > c->task_cap || (size_t)c->n_lm > c->lm_cap || c->n_recs > c->rec_cap))
    rc = fail(c, MK_ERR_UNSUPPORTED, "re-partitioned graph exceeds the workspace reserve");
  if (rc != MK_OK) {
    std::string m = c->err;
    c->sm_weights = old;
    for (int k = 0; k < 8; ++k) c->op_weights[k] = old_op[k];
    c->g = old_g;
    c->qbegin = old_q;
    c->n_lm = old_lm;
    c->n_recs = old_recs;
    c->weight_bytes_per_step = old_wb;
    return fail(c, rc, m);
  }
  if (c->loaded && upload_graph(c, c->ws) != MK_OK) return MK_ERR_CUDA;
  return MK_OK;
}
}  // namespace

int mk_set_sm_weights(mk_ctx* c, const float* weights, int n, void* stream) {
  return set_weights(c, 0, weights, n, stream);
}

int mk_set_op_sm_weights(mk_ctx* c, int op_kind, const float* weights, int n, void* stream) {
  if (op_kind == 0) return fail(c, MK_ERR_INVALID_ARG, "op_kind must be a projection task kind");
  return set_weights(c, op_kind, weights, n, stream);
}

int mk_set_dispatch(mk_ctx* c, int mode, int tasks_per_sm, void* stream) {
  if (!c) return fail(nullptr, MK_ERR_INVALID_ARG, "ctx is NULL");
  if (!c->tp_shards.empty()) return fail(c, MK_ERR_UNSUPPORTED, "tensor-parallel graphs use static queues");
  if (mode != MK_DISPATCH_STATIC && mode != MK_DISPATCH_CLAIM && mode != MK_DISPATCH_CLAIM_PACED &&
      mode != MK_DISPATCH_CLAIM_PRIORITY)
    return fail(c, MK_ERR_INVALID_ARG, "unknown mode");
  const bool claim = mode != MK_DISPATCH_STATIC;
  if (claim && (tasks_per_sm < 1 || tasks_per_sm > 4))
    return fail(c, MK_ERR_INVALID_ARG, "tasks_per_sm must be in [1, 4]");
  const mk_config& f = c->cfg;
  int variant = c->variant;
  if (claim) {
    if (c->tc || c->bm != 1)
      return fail(c, MK_ERR_UNSUPPORTED, "run-time claims are built for the batch-1 kernel only");
    variant = find_decode_variant(c->nseg_h, c->rps_h, c->nseg_f, c->rps_f, f.head_dim, c->bm, f.qk_norm, 1);
  } else if (!c->tc) {
    variant = find_decode_variant(c->nseg_h, c->rps_h, c->nseg_f, c->rps_f, f.head_dim, c->bm, f.qk_norm, 0);
  }
  if (variant < 0) return fail(c, MK_ERR_UNSUPPORTED, "no kernel instantiation for this shape and dispatch mode");
  if (c->loaded && !cuda_ok(c, cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)), "stream sync"))
    return MK_ERR_CUDA;
  const int old_dyn = c->dyn, old_split = c->dyn_split;
  Graph old_g = c->g;
  std::vector<uint32_t> old_q = c->qbegin, old_pf = c->pool_first, old_pc = c->pool_count;
  const uint64_t old_wb = c->weight_bytes_per_step;
  c->dyn = mode;
  c->dyn_split = claim ? tasks_per_sm : c->dyn_split;
  int rc = build_graph(c);
  if (rc == MK_OK && (c->g.tasks.size() > c->task_cap || (int)c->pool_first.size() > c->pool_cap))
    rc = fail(c, MK_ERR_UNSUPPORTED, "graph exceeds the workspace reserve");
  if (rc != MK_OK) {
    std::string m = c->err;
    c->dyn = old_dyn;
    c->dyn_split = old_split;
    c->g = old_g;
    c->qbegin = old_q;
    c->pool_first = old_pf;
    c->pool_count = old_pc;
    c->weight_bytes_per_step = old_wb;
    return fail(c, rc, m);
  }
  c->variant = variant;
  if (c->loaded && upload_graph(c, c->ws) != MK_OK) return MK_ERR_CUDA;
  return MK_OK;
}

int mk_set_l2_prefetch(mk_ctx* c, int stages) {
  if (!c || stages < 0 || stages > 64) return fail(c, MK_ERR_INVALID_ARG, "stages must be in [0, 64]");
  c->l2_ahead = stages;
  return MK_OK;
}

int mk_set_attn_chunk_keys(mk_ctx* c, int keys) {
  if (!c || keys < 1 || keys > (1 << 20)) return fail(c, MK_ERR_INVALID_ARG, "keys must be in [1, 2^20]");
  c->min_chunk_keys = keys;
  return MK_OK;
}

int mk_set_attn_head_keys(mk_ctx* c, int keys) {
  if (!c || keys < 0 || keys > (1 << 20)) return fail(c, MK_ERR_INVALID_ARG, "keys must be in [0, 2^20]");
  c->head_keys = keys;
  return MK_OK;
}

int mk_set_trace(mk_ctx* c, void* device_buffer) {
  if (!c) return fail(nullptr, MK_ERR_INVALID_ARG, "ctx is NULL");
  if (!c->tp_shards.empty()) return fail(c, MK_ERR_UNSUPPORTED, "no tracing of tensor-parallel launches");
  if (device_buffer && (reinterpret_cast<uintptr_t>(device_buffer) & 7))
    return fail(c, MK_ERR_INVALID_ARG, "trace buffer must be 8-byte aligned");
  c->trace = static_cast<uint64_t*>(device_buffer);
  return MK_OK;
}

int mk_get_graph_info(const mk_ctx* c, mk_graph_info* out) {
  if (!c || !out) return MK_ERR_INVALID_ARG;
  out->n_sms = c->n_sms;
  out->n_tasks = (int)c->g.tasks.size();
  out->task_capacity = (int)c->task_cap;
  if (!c->tp_shards.empty()) {  // emulated tensor parallel: every rank's tasks, rank 0's SMs first
    out->n_sms = c->tp_ranks * c->tp_sms;
    out->n_tasks = out->task_capacity = (int)c->tp_tasks.size();
  }
  out->n_events = c->n_events;
  out->attn_chunks = c->nch;
  out->kernel_variant = c->variant;
  out->weight_bytes_per_step = c->weight_bytes_per_step;
  out->smem_bytes = decode_smem_bytes(c->variant);
  return MK_OK;
}

int mk_export_taskgraph(const mk_ctx* c, int32_t* tasks, int task_capacity, int32_t* event_counts,
                        int event_capacity) {
  if (!c) return MK_ERR_INVALID_ARG;
  if (!c->tp_shards.empty()) return MK_ERR_UNSUPPORTED;  // mk_export_taskgraph_tp
  std::vector<VTask> v = to_vtasks(c->g);
  if (tasks)
    for (int i = 0; i < (int)v.size() && i < task_capacity; ++i) {
      const VTask& t = v[i];
      int32_t* o = tasks + (size_t)i * 11;
      o[0] = t.kind; o[1] = t.layer; o[2] = t.sm; o[3] = t.row0; o[4] = t.nrows; o[5] = t.n_wait;
      o[6] = t.wait[0]; o[7] = t.wait[1]; o[8] = t.n_notify; o[9] = t.notify[0]; o[10] = t.notify[1];
    }
  if (event_counts)
    for (int e = 0; e < c->n_events && e < event_capacity; ++e) event_counts[e] = (int32_t)c->g.ev_count[e];
  return (int)v.size();
}

int mk_validate_taskgraph(mk_ctx* c, const int32_t* tasks, int n_tasks, const int32_t* event_counts, int n_events) {
  if (!c || !tasks || !event_counts || n_tasks < 0 || n_events != c->n_events)
    return fail(c, MK_ERR_INVALID_ARG, "bad arguments to mk_validate_taskgraph");
  std::vector<VTask> v(n_tasks);
  for (int i = 0; i < n_tasks; ++i) {
    const int32_t* o = tasks + (size_t)i * 11;
    v[i] = VTask{o[0], o[1], o[2], o[3], o[4], o[5], {o[6], o[7]}, o[8], {o[9], o[10]}};
  }
  std::vector<uint32_t> cnt(n_events);
  for (int e = 0; e < n_events; ++e) cnt[e] = (uint32_t)std::max(0, event_counts[e]);
  return validate(c, v, cnt);
}

size_t mk_attention_workspace_bytes(int BH, int d, int L) {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return attention_workspace_bytes(BH, d, L, n);
}

int mk_attention_decode(const uint16_t* q, const uint16_t* k_t, const uint16_t* v, float* o, int BH, int d, int L,
                        float scale, void* workspace, void* stream) {
  if (!q || !k_t || !v || !o) return fail(nullptr, MK_ERR_INVALID_ARG, "NULL operand");
  if (BH < 1 || L < 1 || (d != 64 && d != 128)) return fail(nullptr, MK_ERR_INVALID_ARG, "bad BH, d or L");
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return fail(nullptr, MK_ERR_CUDA, "no CUDA device");
  std::string err;
  int rc = attention_decode(q, k_t, v, o, BH, d, L, scale, workspace, reinterpret_cast<cudaStream_t>(stream), n,
                            nullptr, &err);
  if (rc) return fail(nullptr, rc, err);
  return MK_OK;
}

int mk_attention_decode_noalloc(const uint16_t* q, const uint16_t* k_t, const uint16_t* v, float* o, int BH, int d,
                                int L, float scale, void* stream) {
  if (!q || !k_t || !v || !o) return fail(nullptr, MK_ERR_INVALID_ARG, "NULL operand");
  if (BH < 1 || L < 1 || (d != 64 && d != 128)) return fail(nullptr, MK_ERR_INVALID_ARG, "bad BH, d or L");
  std::string err;
  int rc = attention_decode_noalloc(q, k_t, v, o, BH, d, L, scale, reinterpret_cast<cudaStream_t>(stream), &err);
  if (rc) return fail(nullptr, rc, err);
  return MK_OK;
}

int mk_attention_status(void* workspace, int BH, int d, int L, void* stream) {
  if (!workspace || BH < 1 || L < 1 || (d != 64 && d != 128)) return fail(nullptr, MK_ERR_INVALID_ARG, "bad arguments");
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return fail(nullptr, MK_ERR_CUDA, "stream sync failed");
  if (L % 8 != 0) return MK_OK;  // the plain-load path has no waits and no workspace
  int dev = 0, n = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  uint32_t* word = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) +
                                               attention_error_word_offset(BH, d, L, n));
  uint32_t e = 0;
  if (cudaMemcpy(&e, word, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return fail(nullptr, MK_ERR_CUDA, "read failed");
  if (e == 0) return MK_OK;
  // a timed-out call may leave arrival counts behind: clear them with the error word
  size_t bytes = attention_workspace_bytes(BH, d, L, n);
  cudaMemset(workspace, 0, bytes);
  cudaDeviceSynchronize();
  return fail(nullptr, MK_ERR_DEVICE_TIMEOUT, "attention wait timed out");
}

int mk_attention_noalloc_status(void* stream) {
  std::string err;
  const int rc = attention_noalloc_status(reinterpret_cast<cudaStream_t>(stream), &err);
  if (rc) return fail(nullptr, rc, err);
  return MK_OK;
}

int mk_attention_set_wait_timeout_ns(uint64_t ns) {
  if (ns == 0) return fail(nullptr, MK_ERR_INVALID_ARG, "the wait limit must be > 0");
  attention_set_wait_timeout_ns(ns);
  return MK_OK;
}

int mk_attention_debug_drop_unit(int unit) {
  attention_debug_drop_unit(unit < 0 ? -1 : unit);
  return MK_OK;
}

int mk_build_taskgraph_tp(const mk_config* cfg, int n_ranks, int device, mk_ctx** out) {
  if (!out) return fail(nullptr, MK_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  std::string why;
  int rc = check_config(cfg, &why);
  if (rc) return fail(nullptr, rc, why);
  const mk_config& f = *cfg;
  const int R = n_ranks;
  if (R < 2 || R > kMaxTpRanks) return fail(nullptr, MK_ERR_INVALID_ARG, "n_ranks must be in [2, 4]");
  if (f.max_batch != 1) return fail(nullptr, MK_ERR_UNSUPPORTED, "tensor parallel serves one sequence (max_batch 1)");
  if (f.qk_norm) return fail(nullptr, MK_ERR_UNSUPPORTED, "no tensor-parallel QK-norm");
  if (f.n_kv_heads % R || f.ffn % (8 * R) || f.vocab % R)
    return fail(nullptr, MK_ERR_INVALID_ARG, "n_kv_heads, ffn / 8 and vocab must divide by n_ranks");
  mk_ctx* c = new mk_ctx();
  c->cfg = f;
  c->device = device;
  if (device >= 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device) != cudaSuccess) {
      delete c;
      return fail(nullptr, MK_ERR_CUDA, "cudaDeviceGetAttribute failed");
    }
    c->n_sms = n;
  } else {
    c->n_sms = 148;
  }
  c->tp_ranks = R;
  c->tp_sms = c->n_sms / R;
  for (int r = 0; r < R; ++r) {
    mk_ctx* sh = new mk_ctx();
    c->tp_shards.push_back(sh);
    sh->cfg = f;
    sh->cfg.n_q_heads /= R;
    sh->cfg.n_kv_heads /= R;
    sh->cfg.ffn /= R;
    sh->cfg.vocab /= R;
    sh->device = device;
    sh->n_sms = c->tp_sms;
    sh->tp_ranks = R;
    sh->tp_rank = r;
    sh->tp_vbase = r * sh->cfg.vocab;
    sh->tp_vfull = f.vocab;
    rc = init_ctx(sh);
    if (rc == MK_OK && sh->variant < 0)
      rc = fail(sh, MK_ERR_UNSUPPORTED, "no tensor-parallel kernel instantiation for this shape");
    if (rc) {
      std::string m = "rank " + std::to_string(r) + ": " + sh->err;
      delete c;
      return fail(nullptr, rc, m);
    }
  }
  // every rank's queues, rank r's SM s at global SM r * tp_sms + s
  c->tp_qbegin.assign((size_t)R * c->tp_sms + 1, 0);
  for (int r = 0; r < R; ++r) {
    const mk_ctx* sh = c->tp_shards[r];
    for (int s2 = 0; s2 < sh->n_sms; ++s2) {
      c->tp_qbegin[(size_t)r * c->tp_sms + s2] = (uint32_t)c->tp_tasks.size();
      for (uint32_t i = sh->qbegin[s2]; i < sh->qbegin[s2 + 1]; ++i) {
        c->tp_tasks.push_back(sh->g.tasks[i].t);
        c->tp_task_sm.push_back(r * c->tp_sms + s2);
      }
    }
    c->weight_bytes_per_step += sh->weight_bytes_per_step;
  }
  c->tp_qbegin[(size_t)R * c->tp_sms] = (uint32_t)c->tp_tasks.size();
  c->n_events = c->tp_shards[0]->n_events;
  rc = validate_tp(c, tp_vtasks(c), c->tp_shards[0]->g.ev_count);
  if (rc) {
    std::string m = c->err;
    delete c;
    return fail(nullptr, rc, m);
  }
  // buffers: the ranks' regions one after another
  for (int r = 0; r < R; ++r) {
    const mk_ctx* sh = c->tp_shards[r];
    c->tp_arena_off.push_back(c->arena_bytes);
    c->arena_bytes = align256(c->arena_bytes + sh->arena_bytes);
    c->tp_kv_off.push_back(c->kv_bytes);
    c->kv_bytes = align256(c->kv_bytes + sh->kv_bytes);
  }
  size_t ws = 0;
  c->tp_ws_tasks = ws;
  ws = align256(ws + c->tp_tasks.size() * sizeof(Task));
  c->tp_ws_qbegin = ws;
  ws = align256(ws + c->tp_qbegin.size() * 4);
  for (int r = 0; r < R; ++r) {
    c->tp_ws_off.push_back(ws);
    ws = align256(ws + c->tp_shards[r]->ws_bytes);
  }
  c->ws_bytes = ws;
  c->variant = c->tp_shards[0]->variant;
  c->nch = c->tp_shards[0]->nch;
  c->bm = 1;
  c->pos.assign(1, 0);
  *out = c;
  return MK_OK;
}

int mk_export_taskgraph_tp(const mk_ctx* c, int32_t* tasks, int task_capacity, int32_t* event_counts,
                           int event_capacity) {
  if (!c || c->tp_shards.empty()) return MK_ERR_INVALID_ARG;
  const std::vector<TVTask> v = tp_vtasks(c);
  if (tasks)
    for (int i = 0; i < (int)v.size() && i < task_capacity; ++i) {
      const TVTask& t = v[i];
      int32_t* o = tasks + (size_t)i * 15;
      o[0] = t.rank; o[1] = t.kind; o[2] = t.layer; o[3] = t.sm; o[4] = t.row0; o[5] = t.nrows; o[6] = t.n_wait;
      o[7] = t.wait[0]; o[8] = t.wait[1]; o[9] = t.n_notify; o[10] = t.notify[0]; o[11] = t.notify[1];
      o[12] = t.remote; o[13] = t.mlo; o[14] = t.mhi;
    }
  const auto& cnt = c->tp_shards[0]->g.ev_count;
  if (event_counts)
    for (int e = 0; e < (int)cnt.size() && e < event_capacity; ++e) event_counts[e] = (int32_t)cnt[e];
  return (int)v.size();
}

int mk_validate_taskgraph_tp(mk_ctx* c, const int32_t* tasks, int n_tasks, const int32_t* event_counts, int n_events) {
  if (!c || c->tp_shards.empty() || !tasks || !event_counts || n_tasks < 0)
    return fail(c, MK_ERR_INVALID_ARG, "bad arguments to mk_validate_taskgraph_tp");
  std::vector<TVTask> v(n_tasks);
  for (int i = 0; i < n_tasks; ++i) {
    const int32_t* o = tasks + (size_t)i * 15;
    v[i] = TVTask{o[0], o[1], o[2], o[3], o[4], o[5], o[6], {o[7], o[8]}, o[9], {o[10], o[11]}, o[12], o[13], o[14]};
  }
  std::vector<uint32_t> cnt(n_events);
  for (int e = 0; e < n_events; ++e) cnt[e] = (uint32_t)std::max(0, event_counts[e]);
  return validate_tp(c, v, cnt);
}

const char* mk_last_error(const mk_ctx* c) { return c ? c->err.c_str() : g_err.c_str(); }

void mk_destroy(mk_ctx* c) { delete c; }

}  // extern "C"

// KV-aware admission of requests to one rollout replica (host code): the iteration model
// and the AIMD rule declared with s3r_sched_simulate in s3r.h ([News] summary; [Explainer]
// Jargon, AIMD scheduler, and "Where it earns its keep"; [Wispaper] "dense verification
// still needs the complete KV cache").
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <deque>
#include <vector>

#include "../../include/s3r.h"

namespace {

constexpr int64_t kPageTokens = 16;

int64_t pages_of(int64_t prompt, int64_t generated) {
  return (prompt + generated + kPageTokens - 1) / kPageTokens;
}

bool finite_nonneg(double x) { return std::isfinite(x) && x >= 0.0; }

}  // namespace

extern "C" int s3r_sched_simulate(const s3r_sched_config* cfg, int32_t num_requests,
                                  const int32_t* prompt_len, const int32_t* resp_len,
                                  const uint8_t* tau, int64_t tau_stride, const int32_t* pressure,
                                  int64_t pressure_len, s3r_sched_result* out, int32_t* trace,
                                  int64_t trace_cap) {
  if (!cfg || !out || num_requests < 0 || (num_requests > 0 && (!prompt_len || !resp_len || !tau)))
    return S3R_ERR_INVALID_ARG;
  if (cfg->capacity < 1 || (cfg->policy != 0 && cfg->policy != 1) || (cfg->evict != 0 && cfg->evict != 1))
    return S3R_ERR_INVALID_ARG;
  if (cfg->cap_min < 1 || cfg->cap0 < cfg->cap_min || cfg->cap_max < cfg->cap0 || cfg->max_iters < 0)
    return S3R_ERR_INVALID_ARG;
  const double params[] = {cfg->u_low, cfg->u_high, cfg->b_high, cfg->c0, cfg->c_tok,
                           cfg->c_kv, cfg->c_xfer, cfg->c_rec, cfg->c_pre};
  for (double x : params)
    if (!finite_nonneg(x)) return S3R_ERR_INVALID_ARG;
  if (tau_stride < 1 || pressure_len < 0 || (pressure_len > 0 && !pressure) || trace_cap < 0 ||
      (trace_cap > 0 && !trace))
    return S3R_ERR_INVALID_ARG;
  for (int32_t r = 0; r < num_requests; ++r)
    if (prompt_len[r] < 0 || resp_len[r] < 0) return S3R_ERR_INVALID_ARG;
  for (int64_t t = 0; t < pressure_len; ++t)
    if (pressure[t] < 0 || pressure[t] >= cfg->capacity) return S3R_ERR_INVALID_ARG;

  std::memset(out, 0, sizeof(*out));
  const int32_t n = num_requests;
  std::vector<int64_t> gen(n, 0), rounds(n, 0);
  std::vector<int32_t> active, still;
  active.reserve(n);
  still.reserve(n);
  std::deque<int32_t> paused;
  int32_t next_new = 0, done = 0;
  int64_t cap = cfg->cap0;
  auto pages = [&](int32_t r) { return pages_of(prompt_len[r], gen[r]); };

  for (int64_t t = 0; t < cfg->max_iters; ++t) {
    if (done == n) break;
    const int64_t cap_t = cfg->capacity - ((pressure && t < pressure_len) ? pressure[t] : 0);
    // one round of every active request, in admission order
    int64_t tokens_t = 0;
    still.clear();
    for (int32_t r : active) {
      if (rounds[r] >= tau_stride) return S3R_ERR_INVALID_ARG;   // out of draws
      const int64_t e = std::min<int64_t>(tau[(size_t)r * tau_stride + rounds[r]], resp_len[r] - gen[r]);
      rounds[r] += 1;
      gen[r] += e;
      tokens_t += e;
      if (gen[r] >= resp_len[r]) ++done;
      else still.push_back(r);
    }
    active.swap(still);
    int64_t U = 0;
    for (int32_t r : active) U += pages(r);
    // evict the most recently admitted until the resident pages fit
    int64_t xfer = 0, rec = 0, pre = 0;
    bool evicted = false;
    while (U > cap_t && !active.empty()) {
      const int32_t r = active.back();
      active.pop_back();
      const int64_t p = pages(r);
      U -= p;
      evicted = true;
      out->evictions += 1;
      if (cfg->evict == 0) xfer += p;
      paused.push_back(r);
    }
    // AIMD on the concurrency cap
    if (cfg->policy == 0) {
      int64_t B = 0;
      for (int32_t r : paused) B += pages(r);
      if (evicted || (double)U > cfg->u_high * (double)cap_t || (double)B > cfg->b_high * (double)cap_t)
        cap = std::max<int64_t>(cfg->cap_min, cap / 2);
      else if ((int64_t)active.size() >= cap && (double)U < cfg->u_low * (double)cap_t)
        cap = std::min<int64_t>(cfg->cap_max, cap + 1);
    }
    // admission: the paused queue first (restores), then new requests, in order, while they fit
    while ((int64_t)active.size() < cap) {
      int32_t r;
      int64_t p;
      if (!paused.empty()) {
        r = paused.front();
        p = pages(r);
        if (U + p > cap_t) break;
        paused.pop_front();
        if (cfg->evict == 0) xfer += p;
        else rec += p;
      } else if (next_new < n) {
        r = next_new;
        p = pages_of(prompt_len[r], 0);
        if (U + p > cap_t) break;
        ++next_new;
        pre += p;
      } else {
        break;
      }
      active.push_back(r);
      U += p;
    }
    const double time_t = cfg->c0 + cfg->c_tok * (double)tokens_t + cfg->c_kv * (double)U +
                          cfg->c_xfer * (double)xfer + cfg->c_rec * (double)rec +
                          cfg->c_pre * (double)pre;
    out->tokens += tokens_t;
    out->transferred += xfer;
    out->recomputed += rec;
    out->prefilled += pre;
    out->time += time_t;
    out->iterations += 1;
    out->max_active = std::max<int32_t>(out->max_active, (int32_t)active.size());
    if (trace && t < trace_cap) {
      int32_t* row = trace + (size_t)t * 8;
      row[0] = (int32_t)cap;
      row[1] = (int32_t)active.size();
      row[2] = (int32_t)paused.size();
      row[3] = (int32_t)U;
      row[4] = (int32_t)xfer;
      row[5] = (int32_t)rec;
      row[6] = (int32_t)pre;
      row[7] = (int32_t)tokens_t;
    }
    // no progress possible: nothing runs, nothing could be admitted, and no pressure to lift
    if (active.empty() && tokens_t == 0 && done < n && (!paused.empty() || next_new < n) && !evicted &&
        (!pressure || t >= pressure_len)) {
      out->stalled = 1;
      break;
    }
  }
  out->done = done;
  return S3R_OK;
}

// Continuous (iteration-level) batching: a scheduler that plans one decoding
// step at a time over the block manager, and an executor that runs a planned
// step through the cache and decode kernels.
//
// Requests join and leave the batch at every step rather than when a whole
// batch is done ("PagedAttention and Continuous Batching", "Batch by step, not
// by request"; "PagedAttention: The vLLM Paper", "Continuous Batching:
// Request-Level vs. Iteration-Level Scheduling"). When the pool runs short the
// newest request is preempted, by swapping its blocks to host memory or by
// dropping them for recomputation ("Implementation Essentials", block manager).
// Parallel samples fork the prompt's blocks ("Implementation Essentials",
// prefix sharing). The step order, the block counts checked before each action
// and the device order of a step are stated in pa.h.
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <new>
#include <unordered_map>
#include <vector>

#include "block_manager.h"
#include "pa_internal.h"

using pa::fail;

namespace {

constexpr int kRing = 3;  // pinned staging buffers in flight
// PA_SCHED_CASCADE_AUTO takes the cascade when the shared blocks it reads once
// instead of once per member of another request add up to this many bytes:
// about what its two extra launches cost at the copy bandwidth.
constexpr double kCascadeMinSavedBytes = 32.0 * 1024 * 1024;

struct Request {
  int64_t id = 0;
  int prompt_len = 0;
  int output_len = 0;
  int num_samples = 1;
  int64_t arrival = 0;
  int64_t order = 0;  // submission index
  int generated = 0;
  std::vector<int32_t> tokens;  // prompt token ids (admission through the prefix cache)
};

struct Write {
  int64_t request;
  int32_t sample;
  int32_t position;
  int64_t slot;
};

struct Plan {
  int64_t step = 0;
  std::vector<int64_t> finished, preempted, resumed, admitted;
  std::vector<int32_t> preempt_modes;
  std::vector<int64_t> swap_out, swap_in, copies;  // flattened pairs
  std::vector<Write> prefill, writes;
  std::vector<int64_t> batch_request;
  std::vector<int32_t> batch_sample, batch_ctx, tables;
  int max_blocks = 1;
  int max_ctx = 0;
  int64_t cached = 0;  // prompt tokens found in the prefix cache

  void clear() {
    finished.clear();
    preempted.clear();
    resumed.clear();
    admitted.clear();
    preempt_modes.clear();
    swap_out.clear();
    swap_in.clear();
    copies.clear();
    prefill.clear();
    writes.clear();
    batch_request.clear();
    batch_sample.clear();
    batch_ctx.clear();
    tables.clear();
    max_blocks = 1;
    max_ctx = 0;
    cached = 0;
  }
};

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace

struct pa_sched {
  pa_bm* bm = nullptr;
  int block_size = 0;
  int max_num_seqs = 0;
  int mode = PA_PREEMPT_SWAP;
  std::unordered_map<int64_t, Request> requests;
  std::vector<int64_t> pending;    // submitted, not yet arrived (submission order)
  std::vector<int64_t> waiting;    // arrival order
  std::vector<int64_t> swapped;    // arrival order
  std::vector<int64_t> running;    // admission order
  std::vector<int64_t> finishing;  // finished in the last step, freed in the next
  int64_t step_index = 0;
  int64_t submitted = 0;
  bool failed = false;
  bool executed = true;
  Plan plan;

  // executor
  bool attached = false;
  int hq = 0, hkv = 0, head_dim = 0, dtype = 0, max_ctx_cap = 0, max_blocks_cap = 0;
  int cache_dtype = 0;              // dtype, or PA_FP8_E4M3
  float k_scale = 1.f, v_scale = 1.f;
  size_t cap_prefill = 0, cap_tokens = 0, meta_bytes = 0;
  void* dev_meta = nullptr;
  void* host_meta[kRing] = {};
  cudaEvent_t ring_ev[kRing] = {};
  int ring_next = 0;
  void* workspace = nullptr;
  size_t workspace_bytes = 0;
  std::vector<int32_t> order_tmp;
  // decode through the cascade when batch sequences share leading blocks
  int cascade_mode = PA_SCHED_CASCADE_AUTO;
  void* cascade_ws = nullptr;
  size_t cascade_ws_bytes = 0;
  int last_groups = 0;
  int64_t last_saved_blocks = 0;
  std::vector<int64_t> ids_tmp;
  std::vector<int32_t> gm_tmp, gp_tmp, sg_tmp, sm_tmp;

  static int64_t seq_of(int64_t request, int sample) {
    return request * PA_SCHED_MAX_SAMPLES + sample;
  }
  pa_bm::Seq& seq(int64_t request, int sample) { return bm->seqs.at(seq_of(request, sample)); }
  Request& req(int64_t id) { return requests.at(id); }

  void insert_by_arrival(std::vector<int64_t>& q, int64_t id) {
    const Request& r = req(id);
    size_t i = 0;
    while (i < q.size()) {
      const Request& o = req(q[i]);
      if (o.arrival > r.arrival || (o.arrival == r.arrival && o.order > r.order)) break;
      ++i;
    }
    q.insert(q.begin() + i, id);
  }

  int running_seqs() const {
    int n = 0;
    for (int64_t id : running) n += requests.at(id).num_samples;
    return n;
  }

  // Blocks that appending one token to each sample takes, in sample order.
  int64_t append_need(const Request& r) {
    int64_t need = 0;
    std::unordered_map<int32_t, int> taken;
    for (int s = 0; s < r.num_samples; ++s) {
      const pa_bm::Seq& q = seq(r.id, s);
      if (q.len % block_size == 0) {
        ++need;
        continue;
      }
      const int32_t last = q.table.back();
      int& t = taken[last];
      if (bm->ref[last] - t > 1) {
        ++need;
        ++t;
      }
    }
    return need;
  }

  int64_t resume_need(const Request& r) {
    int64_t need = 0;
    for (int s = 0; s < r.num_samples; ++s) {
      const pa_bm::Seq& q = seq(r.id, s);
      need += (int64_t)q.host.size() + (q.len % block_size == 0 ? 1 : 0);
    }
    return need;
  }

  int64_t admit_need(const Request& r) const {
    const int64_t len = (int64_t)r.prompt_len + r.generated;
    const int64_t extra = len % block_size == 0 ? r.num_samples : r.num_samples - 1;
    int hits = 0, revived = 0;
    if (!r.tokens.empty())
      pa_bm_cached_prefix(bm, r.tokens.data(), r.prompt_len, &hits, &revived);
    return ceil_div(len, block_size) - hits + revived + extra;
  }

  int append(const Request& r) {
    for (int s = 0; s < r.num_samples; ++s) {
      const int64_t sid = seq_of(r.id, s);
      const int32_t pos = (int32_t)bm->seqs.at(sid).len;
      int64_t slot = 0, cow[2];
      int n_cow = 0;
      if (int st = pa_bm_append_slots(bm, sid, 1, &slot, cow, &n_cow)) return st;
      if (n_cow) {
        plan.copies.push_back(cow[0]);
        plan.copies.push_back(cow[1]);
      }
      plan.writes.push_back({r.id, s, pos, slot});
    }
    return PA_OK;
  }

  int preempt(int64_t id) {
    const Request& r = req(id);
    size_t host_need = 0;
    for (int s = 0; s < r.num_samples; ++s) host_need += seq(id, s).table.size();
    if (mode == PA_PREEMPT_SWAP && host_need <= bm->host_free.size()) {
      std::vector<int64_t> pairs;
      for (int s = 0; s < r.num_samples; ++s) {
        pairs.resize(2 * seq(id, s).table.size());
        int n = 0;
        if (int st = pa_bm_swap_out(bm, seq_of(id, s), pairs.data(), (int)pairs.size() / 2, &n))
          return st;
        plan.swap_out.insert(plan.swap_out.end(), pairs.begin(), pairs.begin() + 2 * n);
      }
      insert_by_arrival(swapped, id);
      plan.preempted.push_back(id);
      plan.preempt_modes.push_back(PA_PREEMPT_SWAP);
      return PA_OK;
    }
    if (r.num_samples == 1) {
      if (int st = pa_bm_free_seq(bm, seq_of(id, 0))) return st;
      insert_by_arrival(waiting, id);
      plan.preempted.push_back(id);
      plan.preempt_modes.push_back(PA_PREEMPT_RECOMPUTE);
      return PA_OK;
    }
    return fail(PA_ERR_NO_FREE_BLOCKS,
                "request %lld has %d samples and the host pool cannot take its %zu blocks",
                (long long)id, r.num_samples, host_need);
  }

  int step() {
    const int64_t t = step_index;
    plan.clear();
    plan.step = t;
    // arrivals
    std::vector<int64_t> still;
    for (int64_t id : pending) {
      if (req(id).arrival <= t)
        insert_by_arrival(waiting, id);
      else
        still.push_back(id);
    }
    pending.swap(still);
    // (1) free the requests that finished in the last step
    for (int64_t id : finishing) {
      for (int s = 0; s < req(id).num_samples; ++s)
        if (int st = pa_bm_free_seq(bm, seq_of(id, s))) return st;
      plan.finished.push_back(id);
    }
    finishing.clear();
    // (2) running requests append, oldest first; the newest is preempted when short
    size_t i = 0;
    while (i < running.size()) {
      const int64_t id = running[i];
      const int64_t need = append_need(req(id));
      while (need > (int64_t)bm->num_free() && running.back() != id) {
        const int64_t victim = running.back();
        running.pop_back();
        if (int st = preempt(victim)) return st;
      }
      if (need > (int64_t)bm->num_free()) {
        running.pop_back();
        if (int st = preempt(id)) return st;
        break;
      }
      if (int st = append(req(id))) return st;
      ++i;
    }
    if (plan.preempted.empty()) {
      // (3) resume swapped requests in arrival order
      while (!swapped.empty()) {
        Request& r = req(swapped.front());
        if (running_seqs() + r.num_samples > max_num_seqs) break;
        if (resume_need(r) > (int64_t)bm->num_free()) break;
        swapped.erase(swapped.begin());
        std::vector<int64_t> pairs;
        for (int s = 0; s < r.num_samples; ++s) {
          pairs.resize(2 * seq(r.id, s).host.size());
          int n = 0;
          if (int st = pa_bm_swap_in(bm, seq_of(r.id, s), pairs.data(), (int)pairs.size() / 2, &n))
            return st;
          plan.swap_in.insert(plan.swap_in.end(), pairs.begin(), pairs.begin() + 2 * n);
        }
        running.push_back(r.id);
        plan.resumed.push_back(r.id);
        if (int st = append(r)) return st;
      }
      // (4) admit waiting requests in arrival order
      while (swapped.empty() && !waiting.empty()) {
        Request& r = req(waiting.front());
        if (running_seqs() + r.num_samples > max_num_seqs) break;
        if (admit_need(r) > (int64_t)bm->num_free()) break;
        waiting.erase(waiting.begin());
        const int len = r.prompt_len + r.generated;
        std::vector<int64_t> slots(len);
        if (r.tokens.empty()) {
          if (int st = pa_bm_add_seq(bm, seq_of(r.id, 0), len, slots.data())) return st;
          for (int p = 0; p < len; ++p) plan.prefill.push_back({r.id, 0, p, slots[p]});
        } else {
          int cached = 0;
          if (int st = pa_bm_add_seq_cached(bm, seq_of(r.id, 0), r.tokens.data(), r.prompt_len,
                                            slots.data(), &cached))
            return st;
          plan.cached += cached;
          for (int p = cached; p < r.prompt_len; ++p) plan.prefill.push_back({r.id, 0, p, slots[p]});
          if (r.generated) {
            int64_t cow[2];
            int n_cow = 0;
            if (int st = pa_bm_append_slots(bm, seq_of(r.id, 0), r.generated,
                                            slots.data() + r.prompt_len, cow, &n_cow))
              return st;
            for (int i = 0; i < r.generated; ++i)
              plan.prefill.push_back({r.id, 0, r.prompt_len + i, slots[r.prompt_len + i]});
          }
        }
        for (int s = 1; s < r.num_samples; ++s)
          if (int st = pa_bm_fork(bm, seq_of(r.id, 0), seq_of(r.id, s))) return st;
        running.push_back(r.id);
        plan.admitted.push_back(r.id);
        if (int st = append(r)) return st;
      }
    }
    // decode batch; requests reaching their output length finish with this step
    for (int64_t id : running) {
      Request& r = req(id);
      for (int s = 0; s < r.num_samples; ++s) {
        const pa_bm::Seq& q = seq(id, s);
        plan.batch_request.push_back(id);
        plan.batch_sample.push_back(s);
        plan.batch_ctx.push_back((int32_t)q.len);
        plan.max_blocks = std::max(plan.max_blocks, (int)q.table.size());
        plan.max_ctx = std::max(plan.max_ctx, (int)q.len);
      }
      ++r.generated;
    }
    const size_t nb = plan.batch_request.size();
    plan.tables.assign(nb * plan.max_blocks, -1);
    for (size_t b = 0; b < nb; ++b) {
      const pa_bm::Seq& q = seq(plan.batch_request[b], plan.batch_sample[b]);
      std::copy(q.table.begin(), q.table.end(), plan.tables.begin() + b * plan.max_blocks);
    }
    std::vector<int64_t> keep;
    for (int64_t id : running) {
      const Request& r = req(id);
      (r.generated == r.output_len ? finishing : keep).push_back(id);
    }
    running.swap(keep);
    ++step_index;
    executed = false;
    return PA_OK;
  }

  void release_executor() {
    for (int k = 0; k < kRing; ++k) {
      if (ring_ev[k]) {
        cudaEventSynchronize(ring_ev[k]);
        cudaEventDestroy(ring_ev[k]);
        ring_ev[k] = nullptr;
      }
      if (host_meta[k]) {
        cudaFreeHost(host_meta[k]);
        host_meta[k] = nullptr;
      }
    }
    if (dev_meta) cudaFree(dev_meta);
    if (workspace) cudaFree(workspace);
    if (cascade_ws) cudaFree(cascade_ws);
    dev_meta = workspace = cascade_ws = nullptr;
    cascade_ws_bytes = 0;
    attached = false;
  }
};

extern "C" {

int pa_sched_create(int num_blocks, int block_size, const int32_t* initial_free_order,
                    int max_num_seqs, int num_host_blocks, int preempt_mode, pa_sched** out) {
  pa::clear_error();
  if (!out) return fail(PA_ERR_INVALID_ARG, "out must not be NULL");
  *out = nullptr;
  if (max_num_seqs <= 0 || num_host_blocks < 0)
    return fail(PA_ERR_INVALID_ARG, "max_num_seqs must be > 0 and num_host_blocks >= 0");
  if (preempt_mode != PA_PREEMPT_SWAP && preempt_mode != PA_PREEMPT_RECOMPUTE)
    return fail(PA_ERR_INVALID_ARG, "unknown preempt_mode %d", preempt_mode);
  if (preempt_mode == PA_PREEMPT_RECOMPUTE && num_host_blocks)
    return fail(PA_ERR_INVALID_ARG, "recompute mode takes no host pool");
  pa_bm* bm = nullptr;
  if (int st = pa_bm_create(num_blocks, block_size, initial_free_order, &bm)) return st;
  if (num_host_blocks) {
    if (int st = pa_bm_set_host_pool(bm, num_host_blocks)) {
      pa_bm_destroy(bm);
      return st;
    }
  }
  pa_sched* s = new (std::nothrow) pa_sched;
  if (!s) {
    pa_bm_destroy(bm);
    return fail(PA_ERR_INVALID_ARG, "out of host memory");
  }
  s->bm = bm;
  s->block_size = block_size;
  s->max_num_seqs = max_num_seqs;
  s->mode = preempt_mode;
  *out = s;
  return PA_OK;
}

void pa_sched_destroy(pa_sched* s) {
  if (!s) return;
  s->release_executor();
  pa_bm_destroy(s->bm);
  delete s;
}

int pa_sched_submit(pa_sched* s, int64_t request_id, int prompt_len, int output_len,
                    int num_samples, int64_t arrival_step) {
  pa::clear_error();
  if (!s) return fail(PA_ERR_INVALID_ARG, "null scheduler");
  if (request_id < 0 || request_id > (INT64_MAX / PA_SCHED_MAX_SAMPLES) - 1)
    return fail(PA_ERR_INVALID_ARG, "request id %lld out of range", (long long)request_id);
  if (s->requests.count(request_id))
    return fail(PA_ERR_INVALID_ARG, "request %lld exists", (long long)request_id);
  if (prompt_len < 1 || output_len < 1 || num_samples < 1 || num_samples > PA_SCHED_MAX_SAMPLES)
    return fail(PA_ERR_INVALID_ARG, "bad request sizes");
  if ((int64_t)prompt_len + output_len > INT32_MAX)
    return fail(PA_ERR_INVALID_ARG, "request longer than 2^31 tokens");
  if (s->mode == PA_PREEMPT_RECOMPUTE && num_samples != 1)
    return fail(PA_ERR_INVALID_ARG, "recompute mode needs one sample per request");
  const int64_t worst = (int64_t)num_samples * ceil_div((int64_t)prompt_len + output_len,
                                                        s->block_size);
  if (num_samples > s->max_num_seqs || worst > s->bm->num_blocks)
    return fail(PA_ERR_NO_FREE_BLOCKS, "request %lld can never fit", (long long)request_id);
  Request r;
  r.id = request_id;
  r.prompt_len = prompt_len;
  r.output_len = output_len;
  r.num_samples = num_samples;
  r.arrival = arrival_step;
  r.order = s->submitted++;
  s->requests.emplace(request_id, r);
  s->pending.push_back(request_id);
  return PA_OK;
}

int pa_sched_submit_tokens(pa_sched* s, int64_t request_id, const int32_t* prompt_tokens,
                           int prompt_len, int output_len, int num_samples,
                           int64_t arrival_step) {
  if (prompt_len > 0 && !prompt_tokens) {
    pa::clear_error();
    return fail(PA_ERR_INVALID_ARG, "null prompt_tokens");
  }
  if (int st = pa_sched_submit(s, request_id, prompt_len, output_len, num_samples, arrival_step))
    return st;
  s->requests.at(request_id).tokens.assign(prompt_tokens, prompt_tokens + prompt_len);
  return PA_OK;
}

int pa_sched_step(pa_sched* s, pa_sched_plan* plan) {
  const pa::NvtxRange nvtx_range("pa_sched_step");
  pa::clear_error();
  if (!s || !plan) return fail(PA_ERR_INVALID_ARG, "null argument");
  if (s->failed) return fail(PA_ERR_NO_FREE_BLOCKS, "scheduler failed in an earlier step");
  if (int st = s->step()) {
    s->failed = true;
    return st;
  }
  const Plan& p = s->plan;
  plan->step = p.step;
  plan->num_finished = (int)p.finished.size();
  plan->num_preempted = (int)p.preempted.size();
  plan->num_resumed = (int)p.resumed.size();
  plan->num_admitted = (int)p.admitted.size();
  plan->num_swap_out = (int)p.swap_out.size() / 2;
  plan->num_swap_in = (int)p.swap_in.size() / 2;
  plan->num_copies = (int)p.copies.size() / 2;
  plan->num_prefill = (int)p.prefill.size();
  plan->num_writes = (int)p.writes.size();
  plan->num_seqs = (int)p.batch_request.size();
  plan->max_blocks_per_seq = p.max_blocks;
  plan->max_context_len = p.max_ctx;
  int64_t total = 0;
  for (int32_t c : p.batch_ctx) total += c;
  plan->total_context = total;
  plan->num_cached_tokens = p.cached;
  return PA_OK;
}

int pa_sched_idle(const pa_sched* s) {
  if (!s) return -1;
  return s->pending.empty() && s->waiting.empty() && s->running.empty() && s->swapped.empty() &&
         s->finishing.empty();
}

int pa_sched_plan_requests(const pa_sched* s, int64_t* finished, int64_t* preempted,
                           int32_t* preempt_modes, int64_t* resumed, int64_t* admitted) {
  pa::clear_error();
  if (!s) return fail(PA_ERR_INVALID_ARG, "null scheduler");
  const Plan& p = s->plan;
  if (finished) std::copy(p.finished.begin(), p.finished.end(), finished);
  if (preempted) std::copy(p.preempted.begin(), p.preempted.end(), preempted);
  if (preempt_modes) std::copy(p.preempt_modes.begin(), p.preempt_modes.end(), preempt_modes);
  if (resumed) std::copy(p.resumed.begin(), p.resumed.end(), resumed);
  if (admitted) std::copy(p.admitted.begin(), p.admitted.end(), admitted);
  return PA_OK;
}

int pa_sched_plan_pairs(const pa_sched* s, int64_t* swap_out, int64_t* swap_in,
                        int64_t* copies) {
  pa::clear_error();
  if (!s) return fail(PA_ERR_INVALID_ARG, "null scheduler");
  const Plan& p = s->plan;
  if (swap_out) std::copy(p.swap_out.begin(), p.swap_out.end(), swap_out);
  if (swap_in) std::copy(p.swap_in.begin(), p.swap_in.end(), swap_in);
  if (copies) std::copy(p.copies.begin(), p.copies.end(), copies);
  return PA_OK;
}

int pa_sched_plan_writes(const pa_sched* s, int which, int64_t* request, int32_t* sample,
                         int32_t* position, int64_t* slot) {
  pa::clear_error();
  if (!s) return fail(PA_ERR_INVALID_ARG, "null scheduler");
  if (which != 0 && which != 1) return fail(PA_ERR_INVALID_ARG, "which must be 0 or 1");
  const std::vector<Write>& w = which == 0 ? s->plan.prefill : s->plan.writes;
  for (size_t i = 0; i < w.size(); ++i) {
    if (request) request[i] = w[i].request;
    if (sample) sample[i] = w[i].sample;
    if (position) position[i] = w[i].position;
    if (slot) slot[i] = w[i].slot;
  }
  return PA_OK;
}

int pa_sched_plan_batch(const pa_sched* s, int64_t* request, int32_t* sample,
                        int32_t* context_lens, int32_t* block_tables) {
  pa::clear_error();
  if (!s) return fail(PA_ERR_INVALID_ARG, "null scheduler");
  const Plan& p = s->plan;
  if (request) std::copy(p.batch_request.begin(), p.batch_request.end(), request);
  if (sample) std::copy(p.batch_sample.begin(), p.batch_sample.end(), sample);
  if (context_lens) std::copy(p.batch_ctx.begin(), p.batch_ctx.end(), context_lens);
  if (block_tables) std::copy(p.tables.begin(), p.tables.end(), block_tables);
  return PA_OK;
}

int pa_sched_kv_usage(const pa_sched* s, int64_t* filled, int64_t* allocated) {
  pa::clear_error();
  if (!s || !filled || !allocated) return fail(PA_ERR_INVALID_ARG, "null argument");
  std::unordered_map<int32_t, int> fill;
  auto visit = [&](int64_t id) {
    const Request& r = s->requests.at(id);
    for (int sm = 0; sm < r.num_samples; ++sm) {
      const pa_bm::Seq& q = s->bm->seqs.at(pa_sched::seq_of(id, sm));
      for (size_t i = 0; i < q.table.size(); ++i) {
        const int f = (int)std::min<int64_t>(s->block_size, q.len - (int64_t)i * s->block_size);
        int& cur = fill[q.table[i]];
        cur = std::max(cur, f);
      }
    }
  };
  for (int64_t id : s->running) visit(id);
  for (int64_t id : s->finishing) visit(id);
  int64_t f = 0;
  for (const auto& kv : fill) f += kv.second;
  *filled = f;
  *allocated = (int64_t)fill.size() * s->block_size;
  return PA_OK;
}

const pa_bm* pa_sched_block_manager(const pa_sched* s) { return s ? s->bm : nullptr; }

int pa_sched_set_cascade(pa_sched* s, int mode) {
  pa::clear_error();
  if (!s) return fail(PA_ERR_INVALID_ARG, "null scheduler");
  if (mode != PA_SCHED_CASCADE_OFF && mode != PA_SCHED_CASCADE_ON &&
      mode != PA_SCHED_CASCADE_AUTO)
    return fail(PA_ERR_INVALID_ARG, "cascade mode %d", mode);
  s->cascade_mode = mode;
  return PA_OK;
}

int pa_sched_last_cascade(const pa_sched* s, int* num_groups, int64_t* shared_blocks) {
  pa::clear_error();
  if (!s || !num_groups || !shared_blocks) return fail(PA_ERR_INVALID_ARG, "null argument");
  *num_groups = s->last_groups;
  *shared_blocks = s->last_saved_blocks;
  return PA_OK;
}

int pa_sched_attach(pa_sched* s, int num_q_heads, int num_kv_heads, int head_dim, int dtype,
                    int max_context_len) {
  pa::clear_error();
  if (!s) return fail(PA_ERR_INVALID_ARG, "null scheduler");
  if (s->attached) return fail(PA_ERR_INVALID_ARG, "executor already attached");
  if (max_context_len <= 0) return fail(PA_ERR_INVALID_ARG, "max_context_len must be > 0");
  if (dtype != PA_F16 && dtype != PA_BF16)
    return fail(PA_ERR_UNSUPPORTED, "dtype %d", dtype);
  // The default split-KV layout depends on the batch size, and a smaller batch
  // may take shorter partitions, so size the workspace for every batch size and
  // a ladder of context lengths up to the cap.
  size_t ws = 0;
  for (int b = 1; b <= s->max_num_seqs; ++b) {
    for (int64_t c = 16;; c = std::min<int64_t>(2 * c, max_context_len)) {
      size_t bytes = 0;
      if (int st = pa_paged_decode_workspace_size(b, num_q_heads, num_kv_heads, head_dim, (int)c,
                                                  s->block_size, 0, &bytes))
        return st;
      ws = std::max(ws, bytes);
      if (c == max_context_len) break;
    }
  }
  const int64_t maxb = ceil_div(max_context_len, s->block_size);
  // The cascade's workspace, for every batch size and number of groups (at most
  // one per two sequences) over the same ladder of context lengths, each
  // context's blocks all shareable.
  const int gh = num_kv_heads > 0 ? num_q_heads / num_kv_heads : 0;
  size_t cws = 0;
  if (gh >= 1 && gh <= 4 && num_q_heads % num_kv_heads == 0) {
    for (int b = 2; b <= s->max_num_seqs; ++b) {
      for (int64_t c = 16;; c = std::min<int64_t>(2 * c, max_context_len)) {
        const int mb = (int)ceil_div(c, s->block_size);
        for (int ng = 1; ng <= b / 2; ++ng) {
          size_t bytes = 0;
          if (pa_paged_decode_cascade_workspace_size(b, num_q_heads, num_kv_heads, head_dim,
                                                     (int)c, mb, s->block_size, ng, 8 / gh, mb,
                                                     &bytes) == PA_OK)
            cws = std::max(cws, bytes);
        }
        if (c == max_context_len) break;
      }
    }
    pa::clear_error();
  }
  const size_t cap_prefill = (size_t)s->bm->num_blocks * s->block_size;
  const size_t cap_tokens = (size_t)s->max_num_seqs;
  size_t bytes = 8 * (cap_prefill + cap_tokens);
  bytes = align_up(bytes, 16) + 4 * (size_t)s->max_num_seqs * maxb;
  bytes = align_up(bytes, 16) + 4 * 2 * (size_t)s->max_num_seqs;
  // group descriptors: members (<= 8 per group, <= one group per two sequences),
  // prefix lengths, and each sequence's group and slot
  bytes = align_up(bytes, 16) + 4 * (size_t)(4 * s->max_num_seqs + s->max_num_seqs / 2 +
                                             2 * s->max_num_seqs) + 64;
  bytes = align_up(bytes, 256);
  s->hq = num_q_heads;
  s->hkv = num_kv_heads;
  s->head_dim = head_dim;
  s->dtype = dtype;
  s->max_ctx_cap = max_context_len;
  s->max_blocks_cap = (int)maxb;
  s->cap_prefill = cap_prefill;
  s->cap_tokens = cap_tokens;
  s->meta_bytes = bytes;
  cudaError_t e = cudaMalloc(&s->dev_meta, bytes);
  if (e == cudaSuccess && ws) e = cudaMalloc(&s->workspace, ws);
  if (e == cudaSuccess && ws) e = cudaMemset(s->workspace, 0, ws);
  if (e == cudaSuccess && cws) e = cudaMalloc(&s->cascade_ws, cws);
  for (int k = 0; k < kRing && e == cudaSuccess; ++k) {
    e = cudaHostAlloc(&s->host_meta[k], bytes, cudaHostAllocDefault);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&s->ring_ev[k], cudaEventDisableTiming);
  }
  if (e != cudaSuccess) {
    s->release_executor();
    return fail(PA_ERR_CUDA, "executor allocation failed: %s", cudaGetErrorString(e));
  }
  s->workspace_bytes = ws;
  s->cascade_ws_bytes = cws;
  s->cache_dtype = dtype;
  s->attached = true;
  return PA_OK;
}

int pa_sched_attach_fp8(pa_sched* s, int num_q_heads, int num_kv_heads, int head_dim, int dtype,
                        int max_context_len, float k_scale, float v_scale) {
  pa::clear_error();
  if (!(k_scale > 0.f && k_scale <= 3.4028234663852886e38f && v_scale > 0.f &&
        v_scale <= 3.4028234663852886e38f))
    return fail(PA_ERR_INVALID_ARG, "k_scale and v_scale must be finite and positive");
  if (int st = pa_sched_attach(s, num_q_heads, num_kv_heads, head_dim, dtype, max_context_len))
    return st;
  s->cache_dtype = PA_FP8_E4M3;
  s->k_scale = k_scale;
  s->v_scale = v_scale;
  return PA_OK;
}

int pa_sched_execute(pa_sched* s, void* k_cache, void* v_cache, void* host_k, void* host_v,
                     const void* prefill_key, const void* prefill_value, const void* key,
                     const void* value, const void* q, void* out, float scale, int* dev_error,
                     void* stream) {
  const pa::NvtxRange nvtx_range("pa_sched_execute");
  pa::clear_error();
  if (!s) return fail(PA_ERR_INVALID_ARG, "null scheduler");
  if (!s->attached) return fail(PA_ERR_INVALID_ARG, "no executor attached");
  if (s->executed) return fail(PA_ERR_INVALID_ARG, "no planned step left to execute");
  const Plan& p = s->plan;
  const int nb = s->bm->num_blocks, bs = s->block_size, d = s->head_dim, hkv = s->hkv;
  const int nseq = (int)p.batch_request.size();
  if (p.max_ctx > s->max_ctx_cap)
    return fail(PA_ERR_INVALID_ARG, "context %d exceeds the attached cap %d", p.max_ctx,
                s->max_ctx_cap);
  if (p.prefill.size() > s->cap_prefill || p.writes.size() > s->cap_tokens)
    return fail(PA_ERR_INVALID_ARG, "step writes more tokens than the executor holds");
  if ((!p.swap_out.empty() || !p.swap_in.empty()) && (!host_k || !host_v))
    return fail(PA_ERR_INVALID_ARG, "the step swaps blocks but no host pool was given");
  if ((!p.prefill.empty() && (!prefill_key || !prefill_value)) ||
      (!p.writes.empty() && (!key || !value)) || (nseq && (!q || !out)))
    return fail(PA_ERR_INVALID_ARG, "null input for a non-empty part of the step");
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  // Sequences of the batch that hold the same leading blocks (samples forked
  // from one prompt, requests whose prompts were found in the prefix cache) are
  // decoded through the cascade, which reads their shared blocks once.
  int ng = 0, maxp = 0;
  const int gh = s->hq / hkv;
  const int gsz = 8 / gh;  // members stacked per KV head: 8 query heads in all
  s->last_groups = 0;
  s->last_saved_blocks = 0;
  // Blocks are shared across requests only through the prefix cache, so the
  // automatic rule has nothing to gain when no request of the batch came in with
  // its prompt's token ids.
  bool consider = s->cascade_mode == PA_SCHED_CASCADE_ON;
  if (s->cascade_mode == PA_SCHED_CASCADE_AUTO)
    for (int i = 0; i < nseq && !consider; ++i)
      consider = !s->req(p.batch_request[i]).tokens.empty();
  if (consider && s->cascade_ws && nseq >= 2 && gsz >= 2) {
    s->ids_tmp.resize(nseq);
    for (int i = 0; i < nseq; ++i)
      s->ids_tmp[i] = pa_sched::seq_of(p.batch_request[i], p.batch_sample[i]);
    s->gm_tmp.resize((size_t)nseq * gsz);
    s->gp_tmp.resize(nseq);
    s->sg_tmp.resize(nseq);
    s->sm_tmp.resize(nseq);
    if (pa_bm_prefix_groups(s->bm, s->ids_tmp.data(), nseq, gsz, s->gm_tmp.data(),
                            s->gp_tmp.data(), s->sg_tmp.data(), s->sm_tmp.data(), &ng,
                            &maxp) != PA_OK)
      return fail(PA_ERR_INVALID_ARG, "grouping the batch: %s", pa_last_error());
    // Block reads saved per group: (members - 1) x its prefix. The automatic
    // rule counts only members of other requests than the group's first: the
    // samples of one request have equal contexts, so the plain decode's
    // longest-first order runs them side by side and L2 already serves their
    // shared prompt once; requests that share a cached prompt are not adjacent.
    int64_t saved = 0, saved_across = 0;
    for (int g = 0; g < ng; ++g) {
      const int32_t* row = s->gm_tmp.data() + (size_t)g * gsz;
      int m = 0, others = 0;
      for (int j = 0; j < gsz && row[j] >= 0; ++j) {
        ++m;
        bool seen = p.batch_request[row[j]] == p.batch_request[row[0]];
        for (int k = 1; k < j && !seen; ++k)
          seen = p.batch_request[row[k]] == p.batch_request[row[j]];
        others += !seen;
      }
      saved += (int64_t)(m - 1) * s->gp_tmp[g];
      saved_across += (int64_t)others * s->gp_tmp[g];
    }
    const double block_bytes =
        2.0 * hkv * bs * d * (s->cache_dtype == PA_FP8_E4M3 ? 1 : 2);
    if (s->cascade_mode == PA_SCHED_CASCADE_AUTO &&
        saved_across * block_bytes < kCascadeMinSavedBytes)
      ng = 0;
    if (ng) {
      size_t need = 0;
      if (pa_paged_decode_cascade_workspace_size(nseq, s->hq, hkv, d, p.max_ctx, p.max_blocks,
                                                 bs, ng, gsz, maxp, &need) != PA_OK ||
          need > s->cascade_ws_bytes)
        ng = 0;
    }
    pa::clear_error();
    if (ng) {
      s->last_groups = ng;
      s->last_saved_blocks = saved;
    }
  }

  // stage slots, tables, context lengths and the order in one pinned buffer
  const int k = s->ring_next;
  s->ring_next = (k + 1) % kRing;
  cudaError_t e = cudaEventSynchronize(s->ring_ev[k]);
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "%s", cudaGetErrorString(e));
  char* h = static_cast<char*>(s->host_meta[k]);
  size_t off = 0;
  int64_t* slots_prefill = reinterpret_cast<int64_t*>(h + off);
  for (size_t i = 0; i < p.prefill.size(); ++i) slots_prefill[i] = p.prefill[i].slot;
  const size_t off_prefill = off;
  off += 8 * p.prefill.size();
  int64_t* slots_tok = reinterpret_cast<int64_t*>(h + off);
  for (size_t i = 0; i < p.writes.size(); ++i) slots_tok[i] = p.writes[i].slot;
  const size_t off_tok = off;
  off = align_up(off + 8 * p.writes.size(), 16);
  const size_t off_tables = off;
  memcpy(h + off, p.tables.data(), 4 * p.tables.size());
  off = align_up(off + 4 * p.tables.size(), 16);
  const size_t off_ctx = off;
  memcpy(h + off, p.batch_ctx.data(), 4 * (size_t)nseq);
  off += 4 * (size_t)nseq;
  const size_t off_order = off;
  s->order_tmp.resize(nseq);
  // longest first; in a cascade step, by the tokens after each sequence's prefix
  if (nseq && ng)
    pa_cascade_order(p.batch_ctx.data(), s->sg_tmp.data(), s->gp_tmp.data(), ng, nseq,
                     s->order_tmp.data());
  else if (nseq)
    pa_longest_first_order(p.batch_ctx.data(), nseq, s->order_tmp.data());
  memcpy(h + off, s->order_tmp.data(), 4 * (size_t)nseq);
  off += 4 * (size_t)nseq;
  // group descriptors (cascade steps only): members, prefix lengths, group and slot
  const size_t off_gm = off = align_up(off, 16);
  if (ng) {
    memcpy(h + off, s->gm_tmp.data(), 4 * (size_t)ng * gsz);
    off += 4 * (size_t)ng * gsz;
  }
  const size_t off_gp = off;
  if (ng) {
    memcpy(h + off, s->gp_tmp.data(), 4 * (size_t)ng);
    off += 4 * (size_t)ng;
  }
  const size_t off_sg = off;
  if (ng) {
    memcpy(h + off, s->sg_tmp.data(), 4 * (size_t)nseq);
    off += 4 * (size_t)nseq;
  }
  const size_t off_sm = off;
  if (ng) {
    memcpy(h + off, s->sm_tmp.data(), 4 * (size_t)nseq);
    off += 4 * (size_t)nseq;
  }
  char* dm = static_cast<char*>(s->dev_meta);
  if (off) {
    e = cudaMemcpyAsync(dm, h, off, cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, "%s", cudaGetErrorString(e));
  }
  e = cudaEventRecord(s->ring_ev[k], st);
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "%s", cudaGetErrorString(e));
  s->executed = true;

  const int nh = s->bm->num_host_blocks;
  const int cdt = s->cache_dtype;
  const bool fp8 = cdt == PA_FP8_E4M3;
  if (!p.swap_out.empty())
    if (int r = pa_swap_blocks(k_cache, v_cache, nb, host_k, host_v, nh, p.swap_out.data(),
                               (int)p.swap_out.size() / 2, hkv, d, bs, cdt, stream))
      return r;
  if (!p.swap_in.empty())
    if (int r = pa_swap_blocks(host_k, host_v, nh, k_cache, v_cache, nb, p.swap_in.data(),
                               (int)p.swap_in.size() / 2, hkv, d, bs, cdt, stream))
      return r;
  const int64_t row = (int64_t)hkv * d;
  // the cache writes of one token list (prefill or new tokens) in the cache's type
  auto write = [&](const void* kk, const void* vv, size_t off_slots, int n) {
    const int64_t* slots = reinterpret_cast<const int64_t*>(dm + off_slots);
    return fp8 ? pa_reshape_and_cache_fp8(kk, vv, row, row, k_cache, v_cache, slots, n, hkv, d, bs,
                                          nb, s->dtype, s->k_scale, s->v_scale, dev_error, stream)
               : pa_reshape_and_cache(kk, vv, row, row, k_cache, v_cache, slots, n, hkv, d, bs, nb,
                                      s->dtype, dev_error, stream);
  };
  if (!p.prefill.empty())
    if (int r = write(prefill_key, prefill_value, off_prefill, (int)p.prefill.size())) return r;
  if (!p.copies.empty())
    if (int r = pa_copy_blocks(k_cache, v_cache, p.copies.data(), (int)p.copies.size() / 2, hkv, d,
                               bs, nb, cdt, stream))
      return r;
  if (!p.writes.empty())
    if (int r = write(key, value, off_tok, (int)p.writes.size())) return r;
  if (nseq) {
    const int32_t* tables = reinterpret_cast<const int32_t*>(dm + off_tables);
    const int32_t* ctx = reinterpret_cast<const int32_t*>(dm + off_ctx);
    const int32_t* order = reinterpret_cast<const int32_t*>(dm + off_order);
    if (ng) {
      const int32_t* gm = reinterpret_cast<const int32_t*>(dm + off_gm);
      const int32_t* gp = reinterpret_cast<const int32_t*>(dm + off_gp);
      const int32_t* sg = reinterpret_cast<const int32_t*>(dm + off_sg);
      const int32_t* sm = reinterpret_cast<const int32_t*>(dm + off_sm);
      return fp8 ? pa_paged_decode_cascade_fp8(
                       out, q, k_cache, v_cache, tables, p.max_blocks, ctx, order, nseq,
                       p.max_ctx, s->hq, hkv, d, bs, nb, scale, s->k_scale, s->v_scale, gm, gp,
                       sg, sm, ng, gsz, maxp, s->cascade_ws, s->cascade_ws_bytes, dev_error,
                       s->dtype, stream)
                 : pa_paged_decode_cascade(out, q, k_cache, v_cache, tables, p.max_blocks, ctx,
                                           order, nseq, p.max_ctx, s->hq, hkv, d, bs, nb, scale,
                                           gm, gp, sg, sm, ng, gsz, maxp, s->cascade_ws,
                                           s->cascade_ws_bytes, dev_error, s->dtype, stream);
    }
    const int r =
        fp8 ? pa_paged_decode_fp8(out, q, k_cache, v_cache, tables, p.max_blocks, ctx, order, nseq,
                                  p.max_ctx, s->hq, hkv, d, bs, nb, scale, s->k_scale, s->v_scale,
                                  0, s->workspace, s->workspace_bytes, dev_error, s->dtype, stream)
            : pa_paged_decode(out, q, k_cache, v_cache, tables, p.max_blocks, ctx, order, nseq,
                              p.max_ctx, s->hq, hkv, d, bs, nb, scale, 0, s->workspace,
                              s->workspace_bytes, dev_error, s->dtype, stream);
    if (r) return r;
  }
  return PA_OK;
}

}  // extern "C"

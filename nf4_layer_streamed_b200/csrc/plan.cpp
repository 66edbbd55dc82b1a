// Slot plan of the streaming pool: the host-only decisions behind every pool call
// (which slot, hit or fill, wait for the previous reader, which rank reads the layer
// from its host store), and their C export.
//
// The reuse rule is the one the layer-streaming review's bug history asks for (Issue
// #331, "4GB 显存微调 8B 模型是真的"): a slot is refilled only after its reader released
// it, and the fill is ordered after that release.  Among the free slots the least
// recently released one is refilled first, so a layer the previous pass released last
// survives into the next pass (the backward starts on the layers the forward left).
// Under the layer-sharded fetch every rank's plan takes the same decisions from the
// same call sequence, so the owner's broadcasts pair up across ranks; the owner of
// layer l is rank l mod world.
#include <new>

#include "internal.h"

namespace nf4ls {

void SlotPlan::init(int n_layers, int depth) {
  n_layers_ = n_layers;
  s_.assign((size_t)depth, Slot());
  tick_ = 0;
  rank_ = 0;
  world_ = 1;
  shared_ = false;
}

int SlotPlan::find(int layer) const {
  for (int i = 0; i < depth(); ++i)
    if (s_[i].layer == layer) return i;
  return -1;
}

bool SlotPlan::holds_any() const {
  for (const Slot& s : s_)
    if (s.layer >= 0) return true;
  return false;
}

int SlotPlan::victim() const {
  int best = -1;
  for (int i = 0; i < depth(); ++i) {
    const Slot& s = s_[i];
    if (s.acquired || s.pending) continue;
    if (s.layer < 0) return i;
    if (best < 0 || s.release_tick < s_[best].release_tick) best = i;
  }
  return best;
}

int SlotPlan::preview(int layer, PlanStep* st) const {
  *st = PlanStep();
  st->owner = shared_ ? layer % world_ : rank_;
  const int held = find(layer);
  if (held >= 0) {
    st->slot = held;
    st->hit = true;
    return NF4LS_OK;
  }
  const int v = victim();
  if (v < 0) return fail(NF4LS_BUFFER_BUSY, "pool: every slot is acquired or pending (depth %d)", depth());
  st->slot = v;
  st->fill = true;
  st->after_release = s_[v].released;
  st->host_read = st->owner == rank_;
  st->broadcast = shared_;
  return NF4LS_OK;
}

int SlotPlan::issue(int layer, PlanStep* st) {
  NF4_TRY(preview(layer, st));
  if (st->fill) {
    Slot& s = s_[st->slot];
    s.layer = layer;
    s.pending = true;
  }
  return NF4LS_OK;
}

void SlotPlan::mark_acquired(int slot) {
  s_[slot].acquired = true;
  s_[slot].pending = false;
}

int SlotPlan::acquire(int layer, PlanStep* st) {
  NF4_TRY(issue(layer, st));
  if (s_[st->slot].acquired) return fail(NF4LS_BUFFER_BUSY, "stream_prefetch: layer %d is already acquired", layer);
  mark_acquired(st->slot);
  return NF4LS_OK;
}

int SlotPlan::acquired_slot(int layer) const {
  const int i = find(layer);
  return i >= 0 && s_[i].acquired ? i : -1;
}

void SlotPlan::release(int slot) {
  Slot& s = s_[slot];
  s.acquired = false;
  s.released = true;
  s.release_tick = ++tick_;
}

}  // namespace nf4ls

struct nf4ls_plan {
  nf4ls::SlotPlan plan;
};

namespace {

void to_c(const nf4ls::PlanStep& s, nf4ls_plan_step* out) {
  if (!out) return;
  out->slot = s.slot;
  out->hit = s.hit;
  out->fill = s.fill;
  out->after_release = s.after_release;
  out->owner = s.owner;
  out->host_read = s.host_read;
  out->broadcast = s.broadcast;
}

int check_layer(const nf4ls_plan* p, int layer, const char* who) {
  if (!p || layer < 0 || layer >= p->plan.n_layers())
    return nf4ls::fail(NF4LS_INVALID_ARG, "%s: bad plan or layer %d", who, layer);
  return NF4LS_OK;
}

}  // namespace

extern "C" int nf4ls_plan_create(int n_layers, int depth, nf4ls_plan** out) {
  nf4ls::clear_error();
  if (!out || n_layers <= 0 || depth < 2 || depth > 8)
    return nf4ls::fail(NF4LS_INVALID_ARG, "nf4ls_plan_create: n_layers %d, depth %d (2..8)", n_layers, depth);
  nf4ls_plan* p = new (std::nothrow) nf4ls_plan();
  if (!p) return nf4ls::fail(NF4LS_INVALID_ARG, "nf4ls_plan_create: out of host memory");
  p->plan.init(n_layers, depth);
  *out = p;
  return NF4LS_OK;
}

extern "C" int nf4ls_plan_share(nf4ls_plan* p, int rank, int world) {
  nf4ls::clear_error();
  if (!p || world < 1 || rank < 0 || rank >= world)
    return nf4ls::fail(NF4LS_INVALID_ARG, "nf4ls_plan_share: bad argument (rank %d, world %d)", rank, world);
  if (p->plan.holds_any()) return nf4ls::fail(NF4LS_INVALID_ARG, "nf4ls_plan_share: the plan must not hold a layer yet");
  p->plan.share(rank, world);
  return NF4LS_OK;
}

extern "C" int nf4ls_plan_prefetch(nf4ls_plan* p, int layer, nf4ls_plan_step* out) {
  nf4ls::clear_error();
  NF4_TRY(check_layer(p, layer, "nf4ls_plan_prefetch"));
  nf4ls::PlanStep s;
  NF4_TRY(p->plan.issue(layer, &s));
  to_c(s, out);
  return NF4LS_OK;
}

extern "C" int nf4ls_plan_acquire(nf4ls_plan* p, int layer, nf4ls_plan_step* out) {
  nf4ls::clear_error();
  NF4_TRY(check_layer(p, layer, "nf4ls_plan_acquire"));
  nf4ls::PlanStep s;
  NF4_TRY(p->plan.acquire(layer, &s));
  to_c(s, out);
  return NF4LS_OK;
}

extern "C" int nf4ls_plan_release(nf4ls_plan* p, int layer) {
  nf4ls::clear_error();
  NF4_TRY(check_layer(p, layer, "nf4ls_plan_release"));
  const int slot = p->plan.acquired_slot(layer);
  if (slot < 0) return nf4ls::fail(NF4LS_INVALID_ARG, "nf4ls_plan_release: layer %d not acquired", layer);
  p->plan.release(slot);
  return NF4LS_OK;
}

extern "C" int nf4ls_plan_destroy(nf4ls_plan* p) {
  delete p;
  return NF4LS_OK;
}

extern "C" int nf4ls_step_pass_ops(int n_layers, int dir, int32_t* ops, int32_t* layers, int cap, int32_t* n_out) {
  nf4ls::clear_error();
  if (n_layers <= 0 || (dir != 1 && dir != -1) || !n_out || cap < 0 || (cap > 0 && (!ops || !layers)))
    return nf4ls::fail(NF4LS_INVALID_ARG, "nf4ls_step_pass_ops: bad argument");
  int n = 0;
  nf4ls::for_each_pass_op(n_layers, dir, nf4ls::kStepLookahead, [&](int op, int layer) {
    if (n < cap) {
      ops[n] = op;
      layers[n] = layer;
    }
    ++n;
    return NF4LS_OK;
  });
  *n_out = n;
  if (n > cap) return nf4ls::fail(NF4LS_INVALID_ARG, "nf4ls_step_pass_ops: %d operations, room for %d", n, cap);
  return NF4LS_OK;
}

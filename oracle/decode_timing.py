"""Timing harness for the CPU oracle: decode layer-steps of single
(sequence, KV head) units, on one core or on many at once.

Test and benchmark infrastructure only (the benchmark's CPU baseline and its
reference arm use it); it runs the oracle as it stands and adds no
arithmetic of its own.  Workers are plain Python processes
(``python -m oracle.decode_timing``) that import numpy and the oracle only,
so they start quickly and are safe to start from a process that already
uses a GPU.

A unit is described by a plain dict (context, block_tokens, budget_blocks,
head_dim, fetch_cap), its host-KV bit pattern (uint16 [1, 1, N, 2, P, D]),
a list of float64 queries per step ([1, Qn, G, D]) and, for workloads with a
residency loss, a list of bool masks per step ([1, 1, K]); both lists are
walked cyclically.
"""

from __future__ import annotations

import math
import os
import pickle
import sys
import time

import numpy as np

if __package__ in (None, ""):                  # run as a worker: python -m oracle.decode_timing
    __package__ = "oracle"
from . import oasis_oracle as O


class OracleUnit:
    """The oracle driving one (sequence, KV head) unit through decode
    layer-steps: attention over its pool, scores, top-K, plan, gather."""

    def __init__(self, cfg: dict, host_bits: np.ndarray):
        self.cfg = cfg
        kv = O.bf16_bits_to_f64(host_bits)
        self.keys, self.vals = kv[:, :, :, 0], kv[:, :, :, 1]
        self.ctx = np.array([cfg["context"]], dtype=np.int64)
        self.kmin, self.kmax = O.block_summaries(self.keys, self.ctx)   # admission, not timed
        K, P, D = cfg["budget_blocks"], cfg["block_tokens"], cfg["head_dim"]
        self.st = np.full((1, 1, K), -1, np.int32)
        self.lu = np.full((1, 1, K), -1, np.int32)
        self.pool_k = np.zeros((1, 1, K, P, D))
        self.pool_v = np.zeros((1, 1, K, P, D))
        self.scale = 1.0 / math.sqrt(D)

    def step(self, q, t, attend=True, mask=None):
        """One decode layer-step (priming when attend is False); `mask`, when
        given, frees slots after the attention and before the plan (R19)."""
        c = self.cfg
        if attend:
            O.sparse_attention(q, self.pool_k, self.pool_v, self.st, self.ctx, self.scale)
        if mask is not None:
            self.st = O.evict_slots(self.st, mask)
        sc = O.lookahead_scores(q, self.kmin, self.kmax, self.ctx, c["block_tokens"])
        sel, _ = O.select_topk(sc, self.ctx, c["budget_blocks"], c["block_tokens"])
        plan = O.plan_fetch(sel, self.st, self.lu, t, c["fetch_cap"])
        self.pool_k = O.prefetch(self.keys, self.pool_k, plan["fetch_slot"], plan["fetch_block"], plan["n_fetch"])
        self.pool_v = O.prefetch(self.vals, self.pool_v, plan["fetch_slot"], plan["fetch_block"], plan["n_fetch"])
        self.st, self.lu = plan["slot_table"], plan["last_used"]


def _one_blas_thread():
    try:
        from threadpoolctl import threadpool_limits
        return threadpool_limits(limits=1)
    except ImportError:                       # pragma: no cover
        return None


def _unit_inputs(spec):
    """(bits, queries, masks or None) of a unit given as (bits, queries) or
    (bits, queries, masks)."""
    bits, queries = spec[0], spec[1]
    return bits, queries, (spec[2] if len(spec) > 2 else None)


def _step_unit(u: OracleUnit, queries: list, masks, i: int):
    u.step(queries[i % len(queries)], i, mask=None if masks is None else masks[i % len(masks)])


def _prepare(cfg: dict, spec, fill_steps: int) -> OracleUnit:
    bits, queries, masks = _unit_inputs(spec)
    u = OracleUnit(cfg, bits)
    u.step(queries[0], 0, attend=False)                   # priming
    for i in range(1, fill_steps + 1):
        _step_unit(u, queries, masks, i)
    return u


def run_unit(cfg: dict, host_bits: np.ndarray, queries: list, fill_steps: int, timed_steps: int,
             masks: list | None = None) -> list:
    """Seconds of each timed decode layer-step of one unit (BLAS on one
    thread): priming, `fill_steps` untimed steps, then `timed_steps` timed."""
    lim = _one_blas_thread()
    try:
        spec = (host_bits, queries, masks)
        u = _prepare(cfg, spec, fill_steps)
        times = []
        for i in range(fill_steps + 1, fill_steps + 1 + timed_steps):
            t0 = time.perf_counter()
            _step_unit(u, queries, masks, i)
            times.append(time.perf_counter() - t0)
        return times
    finally:
        if lim is not None:
            lim.__exit__(None, None, None)


def usable_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):         # pragma: no cover
        return os.cpu_count() or 1


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:                           # pragma: no cover
        pass
    return "unknown"


def _send(stream, obj):
    data = pickle.dumps(obj, protocol=pickle.HIGHEST_PROTOCOL)
    stream.write(len(data).to_bytes(8, "little"))
    stream.write(data)
    stream.flush()


def _recv(stream):
    head = stream.read(8)
    if len(head) != 8:
        raise EOFError("worker closed its pipe")
    n = int.from_bytes(head, "little")
    data = stream.read(n)
    if len(data) != n:
        raise EOFError("worker closed its pipe")
    return pickle.loads(data)


def _worker() -> int:
    """A group of units in a process of its own: receive them, prime and
    fill each, say ready; then, per start byte, one timed decode layer-step of
    every unit of the group in turn (the seconds of the whole group sent back
    as a float64), until the end byte."""
    inp, out = sys.stdin.buffer, sys.stdout.buffer
    cfg, specs, fill_steps = _recv(inp)
    _one_blas_thread()
    units = [(_prepare(cfg, spec, fill_steps), _unit_inputs(spec)) for spec in specs]
    out.write(b"R")
    out.flush()
    i = fill_steps + 1
    while True:
        c = inp.read(1)
        if c != b"G":
            return 0 if c == b"E" else 1
        t0 = time.perf_counter()
        for u, (_, queries, masks) in units:
            _step_unit(u, queries, masks, i)
        out.write(np.float64(time.perf_counter() - t0).tobytes())
        out.flush()
        i += 1


class UnitPool:
    """Units spread over worker processes (one unit per process, or
    `workers` processes taking the units in turn), stepped together:
    `step()` runs one timed decode layer-step on every unit at once and
    returns the wall time (seconds, the parent's clock from start to the last
    reply) and each process's own time.  A watchdog ends the workers if
    `timeout_s` passes, so no call blocks for longer."""

    def __init__(self, cfg: dict, units: list, fill_steps: int, timeout_s: float = 600.0,
                 workers: int | None = None):
        import subprocess
        import threading
        root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
        env = {**os.environ, "OMP_NUM_THREADS": "1", "OPENBLAS_NUM_THREADS": "1", "MKL_NUM_THREADS": "1"}
        self.procs = []
        self._watchdog = threading.Timer(timeout_s, self._kill)
        self._watchdog.daemon = True
        self._watchdog.start()
        n = len(units) if workers is None else max(1, min(workers, len(units)))
        groups = [units[k::n] for k in range(n)]
        try:
            for _ in groups:
                self.procs.append(subprocess.Popen([sys.executable, "-m", "oracle.decode_timing"], cwd=root,
                                                   env=env, stdin=subprocess.PIPE, stdout=subprocess.PIPE))
            for p, group in zip(self.procs, groups):
                _send(p.stdin, (cfg, group, fill_steps))
            for p in self.procs:
                if p.stdout.read(1) != b"R":
                    raise RuntimeError("an oracle worker did not get ready")
        except BaseException:
            self.close()
            raise

    def _kill(self):                             # only the processes started here
        for p in self.procs:
            if p.poll() is None:
                p.kill()

    def step(self):
        t0 = time.perf_counter()
        for p in self.procs:
            p.stdin.write(b"G")
            p.stdin.flush()
        own = []
        for p in self.procs:
            b = p.stdout.read(8)
            if len(b) != 8:
                raise RuntimeError("an oracle worker stopped")
            own.append(float(np.frombuffer(b, dtype=np.float64)[0]))
        return time.perf_counter() - t0, own

    def close(self):
        self._watchdog.cancel()
        for p in self.procs:
            try:
                if p.poll() is None:
                    p.stdin.write(b"E")
                    p.stdin.flush()
                    p.stdin.close()
                    p.wait(timeout=30)
            except Exception:                    # a worker that already ended
                pass
        self._kill()
        for p in self.procs:
            p.wait()

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()


def run_units_parallel(cfg: dict, units: list, fill_steps: int, timed_steps: int, workers: int,
                       timeout_s: float = 600.0) -> list:
    """The timed steps of every (host_bits, queries[, masks]) unit of `units`, run
    `workers` processes at a time, the processes of a wave stepping together.
    Returns each unit's list of step seconds."""
    results = []
    for w0 in range(0, len(units), workers):
        wave = units[w0:w0 + workers]
        with UnitPool(cfg, wave, fill_steps, timeout_s) as pool:
            per = [pool.step()[1] for _ in range(timed_steps)]
        results += [[per[s][k] for s in range(timed_steps)] for k in range(len(wave))]
    return results


if __name__ == "__main__":
    sys.exit(_worker())

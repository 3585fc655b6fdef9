"""Timing of the oracle on all host cores.

TEST INFRASTRUCTURE, NOT PRODUCT CODE: only the CPU-baseline leg of
``bench.py`` runs it. It holds none of the method's arithmetic.

Each worker is its own interpreter (``python -m oracle.timing JOB``), not a
forked child: the parent that starts them holds a CUDA context. A worker
loads its share of a slot-pool decode from the pickled JOB file, runs the
oracle once as a warm-up, prints ``ready``, reads the common start and end
times (wall clock, seconds since the epoch) from stdin, runs the oracle
single-threaded back to back from the start until a call ends after the end
time, and prints ``{"done": tokens, "finished": time}``.
"""

from __future__ import annotations

import json
import pickle
import sys
import time


def _run(job_path: str) -> None:
    from threadpoolctl import threadpool_limits

    from oracle import gdn as O

    with open(job_path, "rb") as f:
        job = pickle.load(f)
    fn = getattr(O, job["fn"])
    args, kw, per_call = job["args"], job["kw"], int(job["tokens_per_call"])
    with threadpool_limits(limits=1):
        fn(*args, **kw)
        print("ready", flush=True)
        window = json.loads(sys.stdin.readline())
        start, end = float(window["start"]), float(window["end"])
        while time.time() < start:
            time.sleep(0.0005)
        done = 0
        while True:
            fn(*args, **kw)
            done += per_call
            now = time.time()
            if now >= end:
                break
    print(json.dumps({"done": done, "finished": now}), flush=True)


if __name__ == "__main__":
    _run(sys.argv[1])

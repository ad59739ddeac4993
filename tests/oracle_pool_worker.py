"""One worker of the bench's CPU baseline: the oracle over a share of a decode
step, on one host core.

Test infrastructure: started by bench.py's CPU-baseline leg as
``python -m tests.oracle_pool_worker``, one process per core.  It imports
numpy and the oracle only.  Protocol on stdin/stdout: the parent writes one
pickled dict with the share's inputs (its texts' pool blocks, renumbered; q,
k, v, slots, tables, lengths; the (text, head) pairs to compute); the worker
answers ``ready``.  Each ``run`` line then runs the oracle once (the cache
write, then attention over the pairs) and answers ``done``; ``quit`` ends.
"""
import os
import pickle
import sys


def main() -> int:
    os.environ.setdefault("OMP_NUM_THREADS", "1")
    os.environ.setdefault("OPENBLAS_NUM_THREADS", "1")
    os.environ.setdefault("MKL_NUM_THREADS", "1")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    if root not in sys.path:
        sys.path.insert(0, root)
    from threadpoolctl import threadpool_limits

    import oracle

    src, dst = sys.stdin.buffer, sys.stdout
    x = pickle.load(src)
    dst.write("ready\n")
    dst.flush()
    with threadpool_limits(limits=1):
        while True:
            line = src.readline().decode().strip()
            if line != "run":
                break
            if x.get("fp8") is not None:
                ks, vs = x["fp8"]
                kc, vc = oracle.cache_write_fp8(x["k_cache"], x["v_cache"], x["k"], x["v"],
                                                x["slots"], x["block_size"], ks, vs)
                oracle.paged_decode_fp8(x["q"], kc, vc, x["tables"], x["lens"], x["scale"],
                                        x["block_size"], ks, vs, x["pairs"])
            else:
                kc, vc = oracle.cache_write(x["k_cache"], x["v_cache"], x["k"], x["v"],
                                            x["slots"], x["block_size"])
                oracle.paged_decode(x["q"], kc, vc, x["tables"], x["lens"], x["scale"],
                                    x["block_size"], x["pairs"])
            dst.write("done\n")
            dst.flush()
    return 0


if __name__ == "__main__":
    sys.exit(main())

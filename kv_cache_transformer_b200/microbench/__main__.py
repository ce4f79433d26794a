"""Build and run the sm_100a cost microbenchmarks (needs a GPU).

    python -m kv_cache_transformer_b200.microbench [rates|staging]

Each program prints one line per measurement; the decode step's design
(mma.sync linears with full K per CTA, bulk-copied activations, one CTA per
SM) follows from these numbers.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "csrc")
INCLUDE = os.path.join(os.path.dirname(os.path.dirname(HERE)), "include")
BUILD = os.path.join(os.path.dirname(os.path.dirname(HERE)), "_build")


def build(name: str) -> str:
    os.makedirs(BUILD, exist_ok=True)
    exe = os.path.join(BUILD, f"microbench_{name}")
    src = os.path.join(HERE, f"{name}.cu")
    if not os.path.exists(exe) or os.path.getmtime(exe) < os.path.getmtime(src):
        subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-I", CSRC,
                        "-I", INCLUDE, "-o", exe, src], check=True)
    return exe


def main():
    names = sys.argv[1:] or ["rates", "staging"]
    for n in names:
        print(f"== {n}", flush=True)
        subprocess.run([build(n)], check=True)


if __name__ == "__main__":
    main()

"""Write tmem_ops.inc: the tcgen05.ld / tcgen05.st wrappers of the kernels.

Each wrapper moves n consecutive 32-bit TMEM columns of the calling thread's lane
(the 32x32b shape: warp w of a warpgroup reaches lanes 32 (w % 4) .. 32 (w % 4) + 31)
into or out of an array of n registers, and waits for its own load or store
(tcgen05.wait::ld / ::st) before returning; the _async stores leave the wait to a
separate tmem_wait_st_keep call.  The register lists are long, so they are generated
rather than written by hand.

    python gen_tmem_ops.py            # rewrite tmem_ops.inc next to this file
    python gen_tmem_ops.py --stdout   # print it instead
"""

import os
import sys

LOAD_WIDTHS = (16, 32, 64, 128)
STORE_WIDTHS = (16, 32, 64)
ASYNC_STORE_WIDTHS = ()  # none in use: every TMEM store is waited where it is issued

HEADER = ("// tcgen05.ld / tcgen05.st wrappers: one thread per TMEM lane (32x32b shape).\n"
          "// Each wrapper waits for its own load/store before returning, so the registers\n"
          "// are valid when it returns.\n")


def load(n):
    regs = ", ".join(f"%{i}" for i in range(n))
    outs = ", ".join(f'"=r"(r[{i}])' for i in range(n))
    return [f"// {n} consecutive 32-bit TMEM columns of this thread's lane, waited.",
            f"__device__ __forceinline__ void tmem_ld_x{n}(uint32_t taddr, uint32_t (&r)[{n}]) {{",
            f'  asm volatile("tcgen05.ld.sync.aligned.32x32b.x{n}.b32 {{{regs}}}, [%{n}];\\n\\t"',
            '               "tcgen05.wait::ld.sync.aligned;"',
            f"               : {outs}",
            '               : "r"(taddr) : "memory");',
            "}"]


def store(n):
    regs = ", ".join(f"%{i + 1}" for i in range(n))
    ins = ", ".join(f'"r"(r[{i}])' for i in range(n))
    return [f"// store {n} consecutive 32-bit TMEM columns of this thread's lane, waited.",
            f"__device__ __forceinline__ void tmem_st_x{n}(uint32_t taddr, const uint32_t (&r)[{n}]) {{",
            f'  asm volatile("tcgen05.st.sync.aligned.32x32b.x{n}.b32 [%0], {{{regs}}};\\n\\t"',
            '               "tcgen05.wait::st.sync.aligned;"',
            f'               :: "r"(taddr), {ins} : "memory");',
            "}"]


def store_async(n):
    regs = ", ".join(f"%{i + 1}" for i in range(n))
    ins = ", ".join(f'"r"(r[{i}])' for i in range(n))
    return [f"// store {n} consecutive 32-bit TMEM columns of this thread's lane, not waited: pair it with",
            f"// tmem_wait_st_keep{n} on the same registers, which keeps them live until the store is done.",
            f"__device__ __forceinline__ void tmem_st_x{n}_async(uint32_t taddr, const uint32_t (&r)[{n}]) {{",
            f'  asm volatile("tcgen05.st.sync.aligned.32x32b.x{n}.b32 [%0], {{{regs}}};"',
            f'               :: "r"(taddr), {ins} : "memory");',
            "}"]


def wait_store_keep(n):
    ins = ", ".join(f'"r"(r[{i}])' for i in range(n))
    return [f"// wait for this thread's earlier tcgen05.st; the {n} registers of the last one stay live up to here.",
            f"__device__ __forceinline__ void tmem_wait_st_keep{n}(const uint32_t (&r)[{n}]) {{",
            f'  asm volatile("tcgen05.wait::st.sync.aligned;" :: {ins} : "memory");',
            "}"]


def render():
    lines = []
    for n in LOAD_WIDTHS:
        lines += load(n)
    for n in STORE_WIDTHS:
        lines += store(n)
    for n in ASYNC_STORE_WIDTHS:
        lines += store_async(n)
        lines += wait_store_keep(n)
    return HEADER + "\n".join(lines) + "\n"


if __name__ == "__main__":
    text = render()
    if "--stdout" in sys.argv:
        sys.stdout.write(text)
    else:
        with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "tmem_ops.inc"), "w") as f:
            f.write(text)

"""Writes sm100_tmem.cuh: inline-PTX wrappers whose long operand lists are
tedious to type by hand (tcgen05.ld.32x32b.x32 without a wait, and
tcgen05.wait::ld tied to 32 / 64 / 128 registers).

    python gen_tmem_ops.py > /dev/null   (rewrites sm100_tmem.cuh in place)
"""
import os


def ld(n):
    outs = ",".join(f"%{i}" for i in range(n))
    cons = ", ".join(f'"=r"(r[{i}])' for i in range(n))
    return f'''// TMEM load, 32 lanes x 32 bits, {n} consecutive columns per thread, without
// waiting: the registers are valid only after tmem_wait_ld_tie{n if n in (32,64,128) else ''} on them.
__device__ __forceinline__ void tmem_ld{n}_async(uint32_t taddr, uint32_t* r) {{
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x{n}.b32 {{{outs}}}, [%{n}];"
               : {cons}
               : "r"(taddr));
}}
'''


def tie(n):
    cons = ", ".join(f'"+r"(r[{i}])' for i in range(n))
    return f'''// Wait for this thread's outstanding TMEM loads; the {n} registers are tied
// to the wait so that no use of them is scheduled before it.
__device__ __forceinline__ void tmem_wait_ld_tie{n}(uint32_t* r) {{
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : {cons}
               :
               : "memory");
}}
'''


def main():
    hdr = ("// sm100_tmem.cuh -- tcgen05.ld without an implied wait, and waits tied to the\n"
           "// loaded registers, so several TMEM loads can be in flight at once.\n"
           "// (Operand lists written out by gen_tmem_ops.py in this directory.)\n"
           "#pragma once\n#include <cstdint>\n\nnamespace sskip {\n\n"
           + ld(32) + "\n" + tie(32) + "\n" + tie(64) + "\n" + tie(128)
           + "\n}  // namespace sskip\n")
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "sm100_tmem.cuh")
    with open(path, "w") as f:
        f.write(hdr)


if __name__ == "__main__":
    main()

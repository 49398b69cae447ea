"""Writes tmem_ldst.inc: tcgen05.ld / tcgen05.st wrappers with long register lists."""
import os
# generates the tcgen05.ld/st register-list wrappers
def ld(n):
    regs = ",".join(f"%{i}" for i in range(n))
    outs = ", ".join(f'"=r"(r[{i}])' for i in range(n))
    return f'''__device__ __forceinline__ void tmem_ld_32x32b_x{n}(uint32_t taddr, uint32_t* r) {{
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x{n}.b32 {{{regs}}}, [%{n}];"
               : {outs}
               : "r"(taddr));
}}
'''
def st(n):
    regs = ",".join(f"%{i+1}" for i in range(n))
    ins = ", ".join(f'"r"(r[{i}])' for i in range(n))
    return f'''__device__ __forceinline__ void tmem_st_32x32b_x{n}(uint32_t taddr, const uint32_t* r) {{
  asm volatile("tcgen05.st.sync.aligned.32x32b.x{n}.b32 [%0], {{{regs}}};"
               :: "r"(taddr), {ins} : "memory");
}}
'''
def wait(n):
    ops = ", ".join(f'"+r"(r[{i}])' for i in range(n))
    return f'''// Waits for this thread's outstanding TMEM loads. The registers are listed as
// read-write operands so the compiler cannot move their uses above the wait.
__device__ __forceinline__ void tmem_wait_ld_x{n}(uint32_t* r) {{
  asm volatile("tcgen05.wait::ld.sync.aligned;" : {ops} :: "memory");
}}
'''
out = ["// generated register-list wrappers for tcgen05.ld / tcgen05.st (32x32b shape)\n"]
out.append(ld(32)); out.append(st(32)); out.append(wait(32)); out.append(wait(128))
open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "tmem_ldst.inc"), "w").write("\n".join(out))

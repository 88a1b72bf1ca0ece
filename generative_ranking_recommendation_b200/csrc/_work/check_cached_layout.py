import numpy as np
BM=BN=128
def seg_c(s,u): return 4*((s+3)//4)+8*u
def tp_c(T,B): return ((T+8*B+8+BN)+3)//4*4
rng=np.random.default_rng(0)
for trial in range(20000):
    B=int(rng.integers(1,9))
    n=rng.integers(0,700,size=B); m=rng.integers(0,400,size=B)
    if trial%7==0: n[:]=rng.integers(0,5,size=B)
    hoff=np.concatenate([[0],np.cumsum(n)]); coff=np.concatenate([[0],np.cumsum(m)])
    Th,C=int(hoff[-1]),int(coff[-1]); Tp=tp_c(C+Th,B)
    used=np.zeros(Tp,bool)
    for u in range(B):
        hs,cs,nu,mu=int(hoff[u]),int(coff[u]),int(n[u]),int(m[u])
        base=seg_c(hs+cs,u); n4=(nu+3)&~3
        # writes
        for i in range(nu+mu):
            at=base+(i if i<nu else n4+i-nu)
            assert 0<=at<Tp and not used[at]; used[at]=True
        nk=(nu+BN-1)//BN; rb=base+n4-nu
        for t in range((mu+BM-1)//BM):
            q0=nu+t*BM
            a=rb+q0; assert a%4==0 and a+128<=Tp, (a,Tp)
            for j in range(nk):
                kv0=(nk-1-j)*BN; b=base+kv0; assert b%4==0 and b+128<=Tp
            # diag tile terms at rb + q0 (same as rows)
print("ok")

# Emulates prefill_cache_mma_kernel's fragment indexing against the PTX m16n8k16 layout.
import numpy as np
def run(D):
    BT=128; S=D+8; SW=S//2
    rng=np.random.default_rng(0)
    X=rng.standard_normal((BT,D)); P=rng.standard_normal((D,D))
    sX=np.zeros(BT*S); sP=np.zeros(D*S)
    for r in range(BT): sX[r*S:r*S+D]=X[r]
    for c in range(D): sP[c*S:c*S+D]=P[c]
    word=lambda arr,w:(arr[2*w],arr[2*w+1])   # a 32-bit word = two halves
    out=np.zeros((BT,D))
    for warp in range(8):
        m0=warp*16
        acc=np.zeros((32,D//8,4))
        for ks in range(D//16):
            # per lane fragments
            A=np.zeros((16,16)); Bm=np.zeros((D//8,16,8))
            for lane in range(32):
                g,tg=lane>>2,lane&3; kw=ks*8+tg
                af=[word(sX,(m0+g)*SW+kw),word(sX,(m0+g+8)*SW+kw),word(sX,(m0+g)*SW+kw+4),word(sX,(m0+g+8)*SW+kw+4)]
                # PTX A layout: reg0 (row g, cols 2tg,2tg+1), reg1 (row g+8, same cols), reg2 (row g, cols +8), reg3 (row g+8, cols +8)
                A[g,2*tg:2*tg+2]=af[0]; A[g+8,2*tg:2*tg+2]=af[1]; A[g,2*tg+8:2*tg+10]=af[2]; A[g+8,2*tg+8:2*tg+10]=af[3]
                for nt in range(D//8):
                    bf=[word(sP,(nt*8+g)*SW+kw),word(sP,(nt*8+g)*SW+kw+4)]
                    # PTX B layout: reg0 (k=2tg,2tg+1; n=g), reg1 (k=2tg+8,+9; n=g)
                    Bm[nt,2*tg:2*tg+2,g]=bf[0]; Bm[nt,2*tg+8:2*tg+10,g]=bf[1]
            for nt in range(D//8):
                C=A@Bm[nt]   # 16x8
                for lane in range(32):
                    g,tg=lane>>2,lane&3
                    acc[lane,nt]+= [C[g,2*tg],C[g,2*tg+1],C[g+8,2*tg],C[g+8,2*tg+1]]
        # staging: word (m0+g)*SW + nt*4+tg <- (acc0,acc1); row g+8 <- (acc2,acc3)
        stage=np.zeros(BT*S)
        for lane in range(32):
            g,tg=lane>>2,lane&3
            for nt in range(D//8):
                w=(m0+g)*SW+nt*4+tg; stage[2*w:2*w+2]=acc[lane,nt,0:2]
                w=(m0+g+8)*SW+nt*4+tg; stage[2*w:2*w+2]=acc[lane,nt,2:4]
        RV=D//8
        for i in range(16*RV):
            r=m0+i//RV; v=i%RV
            out[r,v*8:v*8+8]=stage[r*S+v*8:r*S+v*8+8]
    err=np.abs(out-X@P.T).max(); print(D, err); assert err<1e-12
    # bank check of the fragment loads
    for base in (0,):
        banks=[((g)*SW+tg)%32 for g in range(8) for tg in range(4)]
        assert len(set(banks))==32
run(64); run(128); print("ok")
